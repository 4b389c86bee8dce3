// Owned-head GQA decode attention with the cache streamed by TMA ("Tensor
// parallel scaling curves", "What tensor parallelism actually splits": each
// shard attends over the heads it owns, with no exchange).
//
// The blocks of kAmKeys cached keys of every (shard, sequence, kv head) pair
// are laid end to end, pair-major, and each CTA (one per SM) takes one
// contiguous range of them ("stream-K"), so every SM streams the same number
// of bytes whatever the batch, head count or cache length.  A range covers
// the tail of one pair, whole pairs and the head of another: each covered
// part of a pair is a "segment".
//
// Per CTA: one producer thread issues 4-D TMA copies of the K and V blocks
// (two 64-dimension boxes each, 128-byte swizzle) into a ring of kAmStages
// stages; two groups of four consumer warps take alternate stages, each warp
// 16 keys of its group's stages, on the tensor cores (mma.sync m16n8k16, bf16
// operands read with ldmatrix from the swizzled tiles): S = Q K^T with the
// g <= 8 query heads of the kv head as rows 0-7 (bf16 hi parts) and 8-15 (lo
// parts), an online softmax per head whose running maximum is raised only when
// a step exceeds it by more than 2^8 (so the output is rarely rescaled), and
// O += P V with P carried the same way.  Two groups keep two warps' dependent
// chains in flight on every SM sub-partition.  At the end of a segment the
// second group's warps hand their state to the first group's (same lanes),
// the first group merges in warp order, the CTA writes its partial (max, sum,
// unnormalised output) for the pair, and the last CTA of the pair to arrive
// (an arrival counter, no waiting) adds the partials in CTA order, then the
// new token's key/value in fp32.  Keys at or past the cache length read as
// zero (the tensor maps end there) and their logits are masked.
//
// The cached keys 0..S-1 are not written by the preceding kernel (it writes
// slot S), so when the new token is given separately the first stages are
// requested before the dependency wait.  Every wait is bounded (2 s); a
// timeout sets the error word, the warps walk on with the work suppressed so
// that every barrier still meets, and the CTA waits (bounded) for its copies
// in flight before it exits.
#pragma once

#include <cuda.h>

#include "tpl_common.cuh"
#include "tpl_gemm.cuh"
#include "tpl_internal.h"

namespace tpl {

constexpr int kAmGroupWarps = 4;                 // warps per consumer group: 16 keys of a stage each
constexpr int kAmGroups = 2;                     // consumer groups, taking alternate stages
constexpr int kAmWarps = kAmGroupWarps * kAmGroups;  // consumer warps; warp kAmWarps is the producer
constexpr int kAmThreads = (kAmWarps + 1) * 32;
constexpr int kAmKeys = 16 * kAmGroupWarps;      // keys per stage, 16 per warp of a group
static_assert(kAmKeys == kAttnTmaKeys, "block size shared with the host geometry");
constexpr int kAmBox = kAmKeys * 64 * 2;         // one box: kAmKeys keys x 64 dims, bf16 (8 KB)
constexpr int kAmStage = 4 * kAmBox;             // K dims 0-63, K dims 64-127, V dims 0-63, V dims 64-127
constexpr int kAmStages = 6;
constexpr int kAmMaxG = 8;
constexpr int kAmMaxCtas = kAttnTmaMaxCtas;      // CTAs per launch at most (bounds the CTAs per pair)
constexpr int kAmMergeBytes = kAmGroupWarps * kAmMaxG * 128 * 4;  // one group's outputs, reused by the pair combine
constexpr int kAmBarBytes = 1024;
constexpr size_t kAmSmem = (size_t)kAmStages * kAmStage + kAmMergeBytes + kAmBarBytes + 1024;
static_assert(kAmSmem <= 232448, "shared memory per block");
constexpr float kAmLazy = 8.0f;  // the running maximum (log2 units) is raised only past this margin

struct AttnTmaArgs {
    CUtensorMap tm_k, tm_v;  // 4-D (128 dims, keys, n_kv/t, t * batch_cap), box (64, kAmKeys, 1, 1)
    const float *q;          // [B][nq][128] fp32
    int B, nq, nkv_s, g, batch_cap;
    int keys;                // cached keys covered (S when the new token is separate, else S + 1)
    int nb;                  // blocks per pair
    int64_t U;               // pairs * nb
    const float *k_new, *v_new;  // [B][n_kv][128] fp32, or NULL
    float scale_log2;
    float *part_o;           // [pairs][cpp_max][g][128]
    float *part_ml;          // [pairs][cpp_max][g][2]
    int cpp_max;
    unsigned *tickets;       // [pairs]
    void *o;                 // [B][nq*128] activation type
    int o_f32;
};

__device__ __forceinline__ void tma_load_4d(void *dst, const CUtensorMap *tm, int x, int y, int z, int w,
                                            uint64_t *bar, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1, {%2, "
        "%3, %4, %5}], [%6], %7;" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(z), "r"(w), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

__device__ __forceinline__ int64_t am_start(int64_t U, int G, int c) { return U * c / G; }

// The CTA whose range holds unit x.
__device__ __forceinline__ int am_cta_of(int64_t U, int G, int64_t x) {
    int c = (int)((x * G) / U);
    while (c > 0 && am_start(U, G, c) > x) --c;
    while (c + 1 < G && am_start(U, G, c + 1) <= x) ++c;
    return c;
}

// Byte offset of 16-byte chunk `chunk` of row `row` in a 128-byte-swizzled box.
__device__ __forceinline__ unsigned am_swz(int row, int chunk) {
    return (unsigned)(row * 128 + ((chunk ^ (row & 7)) << 4));
}

__global__ void __launch_bounds__(kAmThreads, 1) attn_decode_tma_kernel(const __grid_constant__ AttnTmaArgs a) {
    constexpr int D = 128;
    constexpr int NS = kAmStages;
    extern __shared__ __align__(1024) unsigned char am_raw[];
    unsigned char *sm = reinterpret_cast<unsigned char *>(((uintptr_t)am_raw + 1023) & ~(uintptr_t)1023);
    float *s_o = reinterpret_cast<float *>(sm + NS * kAmStage);                  // [kAmWarps][8][128]
    uint64_t *full = reinterpret_cast<uint64_t *>(sm + NS * kAmStage + kAmMergeBytes);
    uint64_t *empty = full + NS;
    float *s_ml = reinterpret_cast<float *>(empty + NS);                         // [kAmWarps][8][2]
    float *s_red = s_ml + kAmWarps * kAmMaxG * 2;                                // [kAmWarps][8]
    float *s_misc = s_red + kAmWarps * kAmMaxG;                                  // M[8], den[8], new[8]
    volatile int *s_flag = reinterpret_cast<volatile int *>(s_misc + 3 * kAmMaxG);  // fail, last, issued
    static_assert(2 * NS * 8 + (kAmWarps * kAmMaxG * 3 + 3 * kAmMaxG) * 4 + 16 <= kAmBarBytes, "barrier area");

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = gridDim.x, cta = blockIdx.x;
    const int64_t u0 = am_start(a.U, G, cta), u1 = am_start(a.U, G, cta + 1);
    const int n = (int)(u1 - u0);
    const bool early = a.k_new != nullptr;
    TPL_TRACE_VARS
    if (threadIdx.x == 0) TPL_TRACE_AT(0);

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kAmGroupWarps);  // the four warps of the stage's group
        }
        s_flag[0] = 0;
        s_flag[1] = 0;
        s_flag[2] = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    pdl_trigger();

    if (warp == kAmWarps) {
        // ---- producer ----
        if (lane == 0) {
            const uint64_t kvpol = evict_first_policy();  // the cache is read once
            auto issue = [&](int i) {
                const int s = i % NS;
                const int64_t u = u0 + i;
                const int pair = (int)(u / a.nb), blk = (int)(u % a.nb);
                const int jl = pair % a.nkv_s, sbB = pair / a.nkv_s;
                const int b = sbB % a.B, sh = sbB / a.B;
                const int sb = sh * a.batch_cap + b;
                unsigned char *st = sm + s * kAmStage;
                mbar_expect_tx(&full[s], kAmStage);
                tma_load_4d(st, &a.tm_k, 0, blk * kAmKeys, jl, sb, &full[s], kvpol);
                tma_load_4d(st + kAmBox, &a.tm_k, 64, blk * kAmKeys, jl, sb, &full[s], kvpol);
                tma_load_4d(st + 2 * kAmBox, &a.tm_v, 0, blk * kAmKeys, jl, sb, &full[s], kvpol);
                tma_load_4d(st + 3 * kAmBox, &a.tm_v, 64, blk * kAmKeys, jl, sb, &full[s], kvpol);
            };
            const int pre = n < NS ? n : NS;
            int i = 0;
            if (early)
                for (; i < pre; ++i) issue(i);
            pdl_wait();
            for (; i < n; ++i) {
                if (i >= NS) {
                    if (s_flag[0] || !mbar_wait(&empty[i % NS], ((unsigned)(i / NS) & 1u) ^ 1u)) {
                        s_flag[0] = 1;
                        break;
                    }
                }
                issue(i);
            }
            s_flag[2] = i;
        }
    } else {
        // ---- consumers: group grp takes the stages i with i % kAmGroups == grp;
        //      warp wl of a group takes keys 16 wl .. 16 wl + 15 of them ----
        pdl_wait();
        if (threadIdx.x == 0) TPL_TRACE_AT(1);
        const int gid = lane >> 2, c = lane & 3;
        const int grp = warp / kAmGroupWarps, wl = warp % kAmGroupWarps;
        const int tid = threadIdx.x;  // group 0: 0..127, one head dimension each in the merge
        bool dead = false;
        int i = 0;
        while (i < n) {
            // one segment: the stages of one pair
            const int64_t ub = u0 + i;
            const int pair = (int)(ub / a.nb);
            const int64_t pe = min(u1, (int64_t)(pair + 1) * a.nb);
            const int seg_n = (int)(pe - ub);
            const int jl = pair % a.nkv_s, sbB = pair / a.nkv_s;
            const int b = sbB % a.B, sh = sbB / a.B;
            const int j = sh * a.nkv_s + jl;  // global kv head
            // q fragments: rows gid (hi) / gid + 8 (lo) of head gid, dims 16ks + 2c (+1, +8, +9)
            uint32_t qf[8][4];
            {
                const bool live = gid < a.g;
                const float *qp = a.q + ((int64_t)b * a.nq + (int64_t)j * a.g + (live ? gid : 0)) * D;
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    float2 u = make_float2(0.f, 0.f), w = make_float2(0.f, 0.f);
                    if (live) {
                        u = *reinterpret_cast<const float2 *>(qp + 16 * ks + 2 * c);
                        w = *reinterpret_cast<const float2 *>(qp + 16 * ks + 2 * c + 8);
                    }
                    const uint32_t h0 = pack_bf16x2(u.x, u.y), h2 = pack_bf16x2(w.x, w.y);
                    qf[ks][0] = h0;
                    qf[ks][1] = pack_bf16x2(u.x - bf16lo(h0), u.y - bf16hi(h0));
                    qf[ks][2] = h2;
                    qf[ks][3] = pack_bf16x2(w.x - bf16lo(h2), w.y - bf16hi(h2));
                }
            }
            float o[16][4];
#pragma unroll
            for (int t = 0; t < 16; ++t) o[t][0] = o[t][1] = o[t][2] = o[t][3] = 0.f;
            float m_a = -INFINITY, l_a = 0.f;
            for (int e = 0; e < seg_n; ++e, ++i) {
                if (i % kAmGroups != grp) continue;
                const int s = i % NS;
                if (!dead)
                    dead = !__all_sync(0xffffffffu, !s_flag[0] && mbar_wait(&full[s], (unsigned)(i / NS) & 1u));
                if (dead) {
                    s_flag[0] = 1;
                    continue;
                }
                const int blk = (int)((u0 + i) % a.nb);
                const int kb = blk * kAmKeys + 16 * wl;  // first key of this warp's 16
                if (kb < a.keys) {
                    const unsigned char *st = sm + s * kAmStage;
                    const unsigned char *Klo = st, *Khi = st + kAmBox, *Vlo = st + 2 * kAmBox,
                                        *Vhi = st + 3 * kAmBox;
                    float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
                    {
                        const int row = 16 * wl + (lane & 7) + ((lane >> 4) << 3);
                        const int half = (lane >> 3) & 1;
#pragma unroll
                        for (int ks = 0; ks < 8; ++ks) {
                            const unsigned char *box = ks < 4 ? Klo : Khi;
                            uint32_t b0, b1, b2, b3;
                            ldsm_x4(box + am_swz(row, 2 * (ks & 3) + half), b0, b1, b2, b3);
                            mma_bf16_16816(s0, qf[ks][0], qf[ks][1], qf[ks][2], qf[ks][3], b0, b1);
                            mma_bf16_16816(s1, qf[ks][0], qf[ks][1], qf[ks][2], qf[ks][3], b2, b3);
                        }
                    }
                    // logits: hi rows + lo rows of the same head; keys kb + 2c, +1 (tile 0), kb + 8 + 2c, +1 (tile 1)
                    const int kk = kb + 2 * c;
                    const float x0 = kk < a.keys ? (s0[0] + s0[2]) * a.scale_log2 : -INFINITY;
                    const float x1 = kk + 1 < a.keys ? (s0[1] + s0[3]) * a.scale_log2 : -INFINITY;
                    const float x2 = kk + 8 < a.keys ? (s1[0] + s1[2]) * a.scale_log2 : -INFINITY;
                    const float x3 = kk + 9 < a.keys ? (s1[1] + s1[3]) * a.scale_log2 : -INFINITY;
                    float mx = fmaxf(fmaxf(x0, x1), fmaxf(x2, x3));
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
                    // mx is finite: key kb is in range.  Raise the running
                    // maximum only past the margin; until then p <= 2^kAmLazy.
                    if (mx > m_a + kAmLazy) {
                        const float alpha = exp2f(m_a - mx);  // 0 on the first step (m_a = -inf)
                        m_a = mx;
                        l_a *= alpha;
#pragma unroll
                        for (int t = 0; t < 16; ++t) {
                            o[t][0] *= alpha;
                            o[t][1] *= alpha;
                            o[t][2] *= alpha;
                            o[t][3] *= alpha;
                        }
                    }
                    const float p0 = exp2f(x0 - m_a), p1 = exp2f(x1 - m_a), p2 = exp2f(x2 - m_a),
                                p3 = exp2f(x3 - m_a);
                    l_a += (p0 + p1) + (p2 + p3);
                    const uint32_t ph0 = pack_bf16x2(p0, p1), ph2 = pack_bf16x2(p2, p3);
                    const uint32_t pl0 = pack_bf16x2(p0 - bf16lo(ph0), p1 - bf16hi(ph0));
                    const uint32_t pl2 = pack_bf16x2(p2 - bf16lo(ph2), p3 - bf16hi(ph2));
                    {
                        const int row = 16 * wl + (lane & 7) + (((lane >> 3) & 1) << 3);
                        const int half = lane >> 4;
#pragma unroll
                        for (int n2 = 0; n2 < 8; ++n2) {
                            const unsigned char *box = n2 < 4 ? Vlo : Vhi;
                            uint32_t v0, v1, v2, v3;
                            ldsm_x4_t(box + am_swz(row, 2 * (n2 & 3) + half), v0, v1, v2, v3);
                            mma_bf16_16816(o[2 * n2], ph0, pl0, ph2, pl2, v0, v1);
                            mma_bf16_16816(o[2 * n2 + 1], ph0, pl0, ph2, pl2, v2, v3);
                        }
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[s]);
            }
            // rows gid + 8 held the P_lo . V half of the same head
#pragma unroll
            for (int t = 0; t < 16; ++t) {
                o[t][0] += o[t][2];
                o[t][1] += o[t][3];
            }
            l_a += __shfl_xor_sync(0xffffffffu, l_a, 1);
            l_a += __shfl_xor_sync(0xffffffffu, l_a, 2);

            // ---- group 1 hands its state to group 0 (warp wl to warp wl, same lanes) ----
            if (grp == 1 && gid < a.g) {
#pragma unroll
                for (int t = 0; t < 16; ++t) {
                    s_o[(wl * kAmMaxG + gid) * D + 8 * t + 2 * c] = o[t][0];
                    s_o[(wl * kAmMaxG + gid) * D + 8 * t + 2 * c + 1] = o[t][1];
                }
                if (c == 0) {
                    s_ml[(wl * kAmMaxG + gid) * 2 + 0] = m_a;
                    s_ml[(wl * kAmMaxG + gid) * 2 + 1] = l_a;
                }
            }
            asm volatile("bar.sync 1, %0;" ::"n"(kAmWarps * 32) : "memory");
            if (grp == 0 && gid < a.g) {
                const float m1 = s_ml[(wl * kAmMaxG + gid) * 2 + 0], l1 = s_ml[(wl * kAmMaxG + gid) * 2 + 1];
                const float M = fmaxf(m_a, m1);
                const float w0 = m_a == -INFINITY ? 0.f : exp2f(m_a - M);
                const float w1 = m1 == -INFINITY ? 0.f : exp2f(m1 - M);
#pragma unroll
                for (int t = 0; t < 16; ++t) {
                    o[t][0] = o[t][0] * w0 + s_o[(wl * kAmMaxG + gid) * D + 8 * t + 2 * c] * w1;
                    o[t][1] = o[t][1] * w0 + s_o[(wl * kAmMaxG + gid) * D + 8 * t + 2 * c + 1] * w1;
                }
                l_a = l_a * w0 + l1 * w1;
                m_a = M;
            }
            asm volatile("bar.sync 1, %0;" ::"n"(kAmWarps * 32) : "memory");
            // ---- group 0 merges its warps (ascending order), then the CTA's partial for the pair ----
            if (grp == 0 && gid < a.g) {
#pragma unroll
                for (int t = 0; t < 16; ++t) {
                    s_o[(wl * kAmMaxG + gid) * D + 8 * t + 2 * c] = o[t][0];
                    s_o[(wl * kAmMaxG + gid) * D + 8 * t + 2 * c + 1] = o[t][1];
                }
                if (c == 0) {
                    s_ml[(wl * kAmMaxG + gid) * 2 + 0] = m_a;
                    s_ml[(wl * kAmMaxG + gid) * 2 + 1] = l_a;
                }
            }
            asm volatile("bar.sync 1, %0;" ::"n"(kAmWarps * 32) : "memory");
            if (grp == 0) {
                const int cf = am_cta_of(a.U, G, (int64_t)pair * a.nb);
                const int cl = am_cta_of(a.U, G, (int64_t)pair * a.nb + a.nb - 1);
                const int n_p = cl - cf + 1;
                const int64_t cbase = ((int64_t)pair * a.cpp_max + (cta - cf)) * a.g;
                for (int hrow = 0; hrow < a.g; ++hrow) {
                    float M = -INFINITY;
#pragma unroll
                    for (int w = 0; w < kAmGroupWarps; ++w) M = fmaxf(M, s_ml[(w * kAmMaxG + hrow) * 2]);
                    float num = 0.f, den = 0.f;
#pragma unroll
                    for (int w = 0; w < kAmGroupWarps; ++w) {
                        const float mi = s_ml[(w * kAmMaxG + hrow) * 2];
                        const float wt = mi == -INFINITY ? 0.f : exp2f(mi - M);
                        num += wt * s_o[(w * kAmMaxG + hrow) * D + tid];
                        den += wt * s_ml[(w * kAmMaxG + hrow) * 2 + 1];
                    }
                    a.part_o[(cbase + hrow) * D + tid] = num;
                    if (tid == 0) {
                        a.part_ml[(cbase + hrow) * 2 + 0] = M;
                        a.part_ml[(cbase + hrow) * 2 + 1] = den;
                    }
                }
                __threadfence();
                asm volatile("bar.sync 2, %0;" ::"n"(kAmGroupWarps * 32) : "memory");
                if (tid == 0) {
                    const unsigned prev = atomicAdd(&a.tickets[pair], 1u);
                    s_flag[1] = prev == (unsigned)(n_p - 1);
                    if (prev >= (unsigned)n_p) record_error(2u);
                }
                asm volatile("bar.sync 2, %0;" ::"n"(kAmGroupWarps * 32) : "memory");
                if (s_flag[1]) {
                    // ---- the last CTA of the pair: partials in CTA order, then the new token ----
                    __threadfence();
                    float *s_mlp = s_o;                        // [n_p][g][2]
                    float *s_w = s_o + 2 * kAmMaxG * 160;      // [n_p][8]
                    float *s_M = s_misc, *s_den = s_misc + kAmMaxG, *s_new = s_misc + 2 * kAmMaxG;
                    const bool has_new = a.k_new != nullptr;
                    for (int x = tid; x < n_p * a.g * 2; x += kAmGroupWarps * 32)
                        s_mlp[x] = __ldcg(&a.part_ml[(int64_t)pair * a.cpp_max * a.g * 2 + x]);
                    if (has_new) {
                        const float kd = a.k_new[((int64_t)b * (a.nq / a.g) + j) * D + tid];
                        for (int hrow = 0; hrow < a.g; ++hrow) {
                            float v = a.q[((int64_t)b * a.nq + (int64_t)j * a.g + hrow) * D + tid] * kd;
#pragma unroll
                            for (int o2 = 16; o2 > 0; o2 >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o2);
                            if (lane == 0) s_red[wl * kAmMaxG + hrow] = v;
                        }
                    }
                    asm volatile("bar.sync 2, %0;" ::"n"(kAmGroupWarps * 32) : "memory");
                    if (tid < a.g) {
                        const int hrow = tid;
                        float nl = -INFINITY;
                        if (has_new) {
                            float v = 0.f;
#pragma unroll
                            for (int w = 0; w < kAmGroupWarps; ++w) v += s_red[w * kAmMaxG + hrow];
                            nl = v * a.scale_log2;
                            s_new[hrow] = nl;
                        }
                        float M = nl;
                        for (int x = 0; x < n_p; ++x) M = fmaxf(M, s_mlp[(x * a.g + hrow) * 2]);
                        float den = 0.f;
                        for (int x = 0; x < n_p; ++x) {
                            const float mi = s_mlp[(x * a.g + hrow) * 2];
                            const float wt = mi == -INFINITY ? 0.f : exp2f(mi - M);
                            s_w[x * kAmMaxG + hrow] = wt;
                            den += wt * s_mlp[(x * a.g + hrow) * 2 + 1];
                        }
                        if (has_new) den += exp2f(nl - M);
                        s_M[hrow] = M;
                        s_den[hrow] = den;
                    }
                    asm volatile("bar.sync 2, %0;" ::"n"(kAmGroupWarps * 32) : "memory");
                    for (int hrow = 0; hrow < a.g; ++hrow) {
                        float num = 0.f;
                        const float *po = a.part_o + ((int64_t)pair * a.cpp_max * a.g + hrow) * D + tid;
#pragma unroll 4
                        for (int x = 0; x < n_p; ++x)
                            num += s_w[x * kAmMaxG + hrow] * __ldcg(po + (int64_t)x * a.g * D);
                        if (has_new)
                            num += exp2f(s_new[hrow] - s_M[hrow]) *
                                   a.v_new[((int64_t)b * (a.nq / a.g) + j) * D + tid];
                        store_act(a.o, a.o_f32, ((int64_t)b * a.nq + (int64_t)j * a.g + hrow) * D + tid,
                                  num / s_den[hrow]);
                    }
                    if (tid == 0) atomicExch(&a.tickets[pair], 0u);
                }
            }
            // the merge area is rewritten by the next segment
            asm volatile("bar.sync 1, %0;" ::"n"(kAmWarps * 32) : "memory");
        }
        if (tid == 0) TPL_TRACE_AT(2);
    }
    __syncthreads();
    if (s_flag[0] && threadIdx.x == 0) {
        record_error(8u);
        // wait (bounded) for the copies still in flight before the CTA exits
        const int issued = s_flag[2];
        for (int x = issued - NS > 0 ? issued - NS : 0; x < issued; ++x)
            mbar_wait(&full[x % NS], (unsigned)(x / NS) & 1u);
    }
    if (threadIdx.x == 0) {
        TPL_TRACE_AT(3);
        TPL_TRACE_PUT(TR_ATTN);
    }
}

}  // namespace tpl
