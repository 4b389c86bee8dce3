// Owned-head GQA decode attention ("Tensor parallel scaling curves", "What
// tensor parallelism actually splits": attention runs on the heads a shard
// owns, with no exchange).  One (shard, sequence, kv head) pair is split over
// its S cached keys into `nsplit` ranges; each warp handles one range with an
// online softmax, the CTA's warps merge their (max, sum, unnormalised output)
// in shared memory, and the last CTA of the pair to arrive (an arrival
// counter, no waiting) combines the CTA partials in ascending order and then
// the new token's key/value in fp32, as the
// projection produced them (when they are not given, position S is read from
// the cache like the others).
//
// Per warp, 16 keys per step on the tensor cores (mma.sync m16n8k16, bf16):
//   S = Q K^T  -- A = the g query heads of the kv head (rows), B = 8 keys;
//                 q and P are each carried as two bf16 parts (hi + lo), in
//                 the otherwise-empty rows 8-15 when g <= 8; the head_dim
//                 index of each 16-wide step is
//                 permuted so that a lane's K operands are the 64 contiguous
//                 bytes K[key][32m + 8c .. +8), m = 0..3;
//   O += P V   -- A = P from the S accumulators (register reuse), B = V with
//                 output column n of tile t mapped to head_dim 16n + t, so a
//                 lane's V operands are 32 contiguous bytes per key.
// K and V are streamed straight from HBM with 16-byte loads, double-buffered:
// the next 16 keys load while the current 16 are processed.
#pragma once

#include "tpl_common.cuh"
#include "tpl_internal.h"

namespace tpl {

struct AttnArgs {
    const float *q;  // [B][nq][128] fp32
    const __nv_bfloat16 *kc, *vc;
    int64_t seq_cap;
    int batch_cap;
    int B, nq, nkv_s, g;
    int64_t keys;  // keys covered by the splits: S (new key given separately) or S + 1
    const float *k_new, *v_new;  // [B][n_kv][128] fp32 of the new token, or NULL
    int nsplit, kps;
    float scale_log2;  // log2(e) / sqrt(head_dim)
    float *part_o;     // [pairs][CTAs per pair][g][128]
    float *part_ml;    // [pairs][CTAs per pair][g][2]
    unsigned *tickets; // [pairs]
    void *o;           // [B][nq*128] activation type
    int o_f32;
};

// The last CTA of a (shard, sequence, kv head) pair: the CTA partials in
// ascending order, then the new token's key/value in fp32, for the g <= MAXG
// heads of the pair; one thread per head dimension (128 threads, named as
// `dim`).  Every global load is issued before the first store: with up to 8
// partials per pair (the usual case) all of them at once, since a load after
// a store of the loop before would wait for it (the compiler cannot rule out
// aliasing), and each round trip to L2 costs about a microsecond at the end
// of the kernel (with more partials, or more than 8 heads, in smaller
// batches).  s_mlp holds the partials' (max, sum) [cpp][g][2]; the other
// shared arrays are scratch.  Run by the CTA's first 128 threads (named
// barrier 1).  With `early` the caller has already written the
// warps' parts of the new token's logits to s_red (attn_new_logits) and
// passes the new value's element as vnew.
template <int MAXG>
__device__ __forceinline__ void attn_pair_combine(const AttnArgs &a, int pair, int cpp, int b, int j, int dim,
                                                  int lane, int warp, const float *s_mlp, float (*s_w)[MAXG],
                                                  float *s_M, float *s_den, float *s_new, float (*s_red)[MAXG],
                                                  bool early = false, float vnew_early = 0.f) {
    constexpr int D = 128;
    const bool has_new = a.k_new != nullptr;
    const int64_t kv_i = ((int64_t)b * (a.nq / a.g) + j) * D + dim;
    const int64_t q0 = ((int64_t)b * a.nq + (int64_t)j * a.g) * D + dim;
    float vnew = vnew_early;
    if (has_new && early) {
        if (threadIdx.x < a.g) {
            float v = 0.f;
#pragma unroll
            for (int w = 0; w < kAttnWarps; ++w) v += s_red[w][threadIdx.x];
            s_new[threadIdx.x] = v * a.scale_log2;
        }
    } else if (has_new) {
        // logits of the new token for the g heads, fp32, fixed-order reduction
        const float kd = a.k_new[kv_i];
        vnew = a.v_new[kv_i];
        float qv[MAXG];
#pragma unroll
        for (int h = 0; h < MAXG; ++h) qv[h] = h < a.g ? a.q[q0 + (int64_t)h * D] : 0.f;
#pragma unroll
        for (int h = 0; h < MAXG; ++h) {
            if (h >= a.g) break;
            float v = qv[h] * kd;
#pragma unroll
            for (int o2 = 16; o2 > 0; o2 >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o2);
            if (lane == 0) s_red[warp][h] = v;
        }
        asm volatile("bar.sync 1, 128;" ::: "memory");
        if (threadIdx.x < a.g) {
            float v = 0.f;
#pragma unroll
            for (int w = 0; w < kAttnWarps; ++w) v += s_red[w][threadIdx.x];
            s_new[threadIdx.x] = v * a.scale_log2;
        }
    }
    asm volatile("bar.sync 1, 128;" ::: "memory");
    if (threadIdx.x < a.g) {
        const int hrow = threadIdx.x;
        float M = has_new ? s_new[hrow] : -INFINITY;
        for (int i = 0; i < cpp; ++i) M = fmaxf(M, s_mlp[(i * a.g + hrow) * 2]);
        float den = 0.f;
        for (int i = 0; i < cpp; ++i) {
            const float mi = s_mlp[(i * a.g + hrow) * 2];
            const float wt = mi == -INFINITY ? 0.f : exp2f(mi - M);
            s_w[i][hrow] = wt;
            den += wt * s_mlp[(i * a.g + hrow) * 2 + 1];
        }
        if (has_new) den += exp2f(s_new[hrow] - M);
        s_M[hrow] = M;
        s_den[hrow] = den;
    }
    asm volatile("bar.sync 1, 128;" ::: "memory");
    const float *po = a.part_o + (int64_t)pair * cpp * a.g * D + dim;  // [cpp][g][D]
    const int64_t ps = (int64_t)a.g * D;
    constexpr int CB = MAXG > 8 ? 4 : 8;  // partials loaded at once per head (registers: MAXG * CB)
    float num[MAXG];
    if (cpp <= CB) {
        float pv[MAXG][CB];
#pragma unroll
        for (int h = 0; h < MAXG; ++h)
#pragma unroll
            for (int i = 0; i < CB; ++i) pv[h][i] = (h < a.g && i < cpp) ? __ldcg(po + i * ps + h * D) : 0.f;
#pragma unroll
        for (int h = 0; h < MAXG; ++h) {
            float n = 0.f;
#pragma unroll
            for (int i = 0; i < CB; ++i)
                if (i < cpp) n += s_w[i][h] * pv[h][i];
            num[h] = n;
        }
    } else {
#pragma unroll
        for (int h = 0; h < MAXG; ++h) {
            float n = 0.f;
            if (h < a.g)
                for (int i = 0; i < cpp; ++i) n += s_w[i][h] * __ldcg(po + i * ps + h * D);
            num[h] = n;
        }
    }
#pragma unroll
    for (int h = 0; h < MAXG; ++h) {
        if (h >= a.g) break;
        float n = num[h];
        if (has_new) n += exp2f(s_new[h] - s_M[h]) * vnew;
        store_act(a.o, a.o_f32, q0 + (int64_t)h * D, n / s_den[h]);
    }
}

// The new token's logits for the pair's g heads, each warp's part of the
// fixed-order sum over the head dimension into s_red[warp][h] (the same
// arithmetic as attn_pair_combine's), computed by every CTA right after the
// dependency wait so that the pair's last CTA finds them ready; returns the
// thread's element of the new value.
template <int MAXG>
__device__ __forceinline__ float attn_new_logits(const AttnArgs &a, int b, int j, int dim, int lane, int warp,
                                                 float (*s_red)[MAXG]) {
    constexpr int D = 128;
    if (!a.k_new) return 0.f;
    const int64_t kv_i = ((int64_t)b * (a.nq / a.g) + j) * D + dim;
    const int64_t q0 = ((int64_t)b * a.nq + (int64_t)j * a.g) * D + dim;
    const float kd = a.k_new[kv_i];
    const float vnew = a.v_new[kv_i];
    float qv[MAXG];
#pragma unroll
    for (int h = 0; h < MAXG; ++h) qv[h] = h < a.g ? a.q[q0 + (int64_t)h * D] : 0.f;
#pragma unroll
    for (int h = 0; h < MAXG; ++h) {
        if (h >= a.g) break;
        float v = qv[h] * kd;
#pragma unroll
        for (int o2 = 16; o2 > 0; o2 >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o2);
        if (lane == 0) s_red[warp][h] = v;
    }
    return vnew;
}

template <bool PACKED>  // PACKED: g <= 8, q/P low parts in rows 8-15
__global__ void __launch_bounds__(kAttnWarps * 32) attn_decode_kernel(const __grid_constant__ AttnArgs a) {
    constexpr int D = 128;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gid = lane >> 2, c = lane & 3;
    const int cpp = a.nsplit / kAttnWarps;  // CTAs per pair
    const int pair = blockIdx.x / cpp, chunk = blockIdx.x % cpp;
    const int split = chunk * kAttnWarps + warp;
    // pair -> (shard s, sequence b, local kv head jl); cache is [t][batch_cap][nkv_s][seq_cap][D]
    const int jl = pair % a.nkv_s;
    const int sb = pair / a.nkv_s;
    const int b = sb % a.B, s = sb / a.B;
    const int j = s * a.nkv_s + jl;  // global kv head
    const int64_t cache_off = (((int64_t)s * a.batch_cap + b) * a.nkv_s + jl) * a.seq_cap * D;
    const __nv_bfloat16 *Kp = a.kc + cache_off;
    const __nv_bfloat16 *Vp = a.vc + cache_off;
    const int64_t k0 = (int64_t)split * a.kps;
    const int64_t k1 = min(a.keys, k0 + a.kps);

    // With the new token given separately the splits read cache positions
    // 0..S-1 only, which the preceding kernel (it writes position S) does not
    // touch: start streaming them before waiting on it.
    const bool early = a.k_new != nullptr;

    // Q operands.  Each query value is carried as a bf16 pair hi + lo
    // (lo = q - hi), so the logits keep ~16 mantissa bits.  With g <= 8 the
    // hi parts fill A rows 0-7 and the lo parts rows 8-15 of the same mma
    // (the rows that would otherwise be zero padding); with g > 8 rows 0-15
    // are heads and hi/lo take two mma.
    constexpr bool packed_rows = PACKED;
    uint32_t qh0[16], ql0[16], qh1[16], ql1[16];  // [m*4 + i]: cols 32m+8c+2i, +1
#pragma unroll
    for (int i = 0; i < 16; ++i) qh0[i] = ql0[i] = qh1[i] = ql1[i] = 0u;
    auto load_q = [&](int row, uint32_t *hi, uint32_t *lo) {
        const float *qp = a.q + ((int64_t)b * a.nq + (int64_t)j * a.g + row) * D;
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            const float4 x0 = *reinterpret_cast<const float4 *>(qp + 32 * m + 8 * c);
            const float4 x1 = *reinterpret_cast<const float4 *>(qp + 32 * m + 8 * c + 4);
            const float v[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const uint32_t h = pack_bf16x2(v[2 * i], v[2 * i + 1]);
                hi[m * 4 + i] = h;
                lo[m * 4 + i] = pack_bf16x2(v[2 * i] - bf16lo(h), v[2 * i + 1] - bf16hi(h));
            }
        }
    };
    // K/V operands of 16 keys: K rows kb+gid (tile 0) and kb+8+gid (tile 1),
    // V rows kb+2c, kb+2c+1, kb+8+2c, kb+9+2c at head_dim 16*gid .. +16.
    struct KV16 {
        uint4 kt0[4], kt1[4], va[2], vb[2], vc2[2], vd[2];
    };
    const uint64_t kvpol = evict_first_policy();  // the cache is read once
    auto load16 = [&](KV16 &f, int64_t kb) {
        const int64_t key0 = kb + gid, key1 = kb + 8 + gid;
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            f.kt0[m] = key0 < k1 ? ldg_stream(Kp + key0 * D + 32 * m + 8 * c, kvpol) : make_uint4(0, 0, 0, 0);
            f.kt1[m] = key1 < k1 ? ldg_stream(Kp + key1 * D + 32 * m + 8 * c, kvpol) : make_uint4(0, 0, 0, 0);
        }
        const int64_t ka = kb + 2 * c, kbb = ka + 1, kc_ = ka + 8, kd = ka + 9;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int col = 16 * gid + 8 * h;
            f.va[h] = ka < k1 ? ldg_stream(Vp + ka * D + col, kvpol) : make_uint4(0, 0, 0, 0);
            f.vb[h] = kbb < k1 ? ldg_stream(Vp + kbb * D + col, kvpol) : make_uint4(0, 0, 0, 0);
            f.vc2[h] = kc_ < k1 ? ldg_stream(Vp + kc_ * D + col, kvpol) : make_uint4(0, 0, 0, 0);
            f.vd[h] = kd < k1 ? ldg_stream(Vp + kd * D + col, kvpol) : make_uint4(0, 0, 0, 0);
        }
    };
    KV16 bufA, bufB;
    TPL_TRACE_VARS
    if (threadIdx.x == 0) TPL_TRACE_AT(0);
    if (early && k0 < k1) load16(bufA, k0);
    pdl_wait();
    pdl_trigger();
    if (threadIdx.x == 0) TPL_TRACE_AT(1);
    if (!early && k0 < k1) load16(bufA, k0);

    if (gid < a.g) load_q(gid, qh0, ql0);
    if constexpr (!PACKED) {
        if (gid + 8 < a.g) load_q(gid + 8, qh1, ql1);
    }

    float o[16][4];
#pragma unroll
    for (int t = 0; t < 16; ++t) o[t][0] = o[t][1] = o[t][2] = o[t][3] = 0.f;
    float m_a = -INFINITY, m_b = -INFINITY;  // running max of rows gid, gid+8 (log2 domain)
    float l_a = 0.f, l_b = 0.f;              // lane-partial running sums

    auto process = [&](const KV16 &f, int64_t kb) {
        const uint4 *kt0 = f.kt0, *kt1 = f.kt1;
        const uint4 *va = f.va, *vb = f.vb, *vc2 = f.vc2, *vd = f.vd;
        // ---- scores: s0 keys kb+2c, +1 (tile 0), s1 keys kb+8+2c, +1 (tile 1) ----
        float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
        if constexpr (PACKED) {
            // rows gid: hi . K, rows gid+8: lo . K (same head)
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                mma_bf16_16816(s0, qh0[m * 4 + 0], ql0[m * 4 + 0], qh0[m * 4 + 1], ql0[m * 4 + 1], kt0[m].x, kt0[m].y);
                mma_bf16_16816(s0, qh0[m * 4 + 2], ql0[m * 4 + 2], qh0[m * 4 + 3], ql0[m * 4 + 3], kt0[m].z, kt0[m].w);
                mma_bf16_16816(s1, qh0[m * 4 + 0], ql0[m * 4 + 0], qh0[m * 4 + 1], ql0[m * 4 + 1], kt1[m].x, kt1[m].y);
                mma_bf16_16816(s1, qh0[m * 4 + 2], ql0[m * 4 + 2], qh0[m * 4 + 3], ql0[m * 4 + 3], kt1[m].z, kt1[m].w);
            }
            s0[0] += s0[2];
            s0[1] += s0[3];
            s1[0] += s1[2];
            s1[1] += s1[3];
            s0[2] = s0[0];
            s0[3] = s0[1];
            s1[2] = s1[0];
            s1[3] = s1[1];
        } else {
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                mma_bf16_16816(s0, qh0[m * 4 + 0], qh1[m * 4 + 0], qh0[m * 4 + 1], qh1[m * 4 + 1], kt0[m].x, kt0[m].y);
                mma_bf16_16816(s0, qh0[m * 4 + 2], qh1[m * 4 + 2], qh0[m * 4 + 3], qh1[m * 4 + 3], kt0[m].z, kt0[m].w);
                mma_bf16_16816(s1, qh0[m * 4 + 0], qh1[m * 4 + 0], qh0[m * 4 + 1], qh1[m * 4 + 1], kt1[m].x, kt1[m].y);
                mma_bf16_16816(s1, qh0[m * 4 + 2], qh1[m * 4 + 2], qh0[m * 4 + 3], qh1[m * 4 + 3], kt1[m].z, kt1[m].w);
                mma_bf16_16816(s0, ql0[m * 4 + 0], ql1[m * 4 + 0], ql0[m * 4 + 1], ql1[m * 4 + 1], kt0[m].x, kt0[m].y);
                mma_bf16_16816(s0, ql0[m * 4 + 2], ql1[m * 4 + 2], ql0[m * 4 + 3], ql1[m * 4 + 3], kt0[m].z, kt0[m].w);
                mma_bf16_16816(s1, ql0[m * 4 + 0], ql1[m * 4 + 0], ql0[m * 4 + 1], ql1[m * 4 + 1], kt1[m].x, kt1[m].y);
                mma_bf16_16816(s1, ql0[m * 4 + 2], ql1[m * 4 + 2], ql0[m * 4 + 3], ql1[m * 4 + 3], kt1[m].z, kt1[m].w);
            }
        }
        const int64_t kk = kb + 2 * c;
        const float x0 = kk < k1 ? s0[0] * a.scale_log2 : -INFINITY;
        const float x1 = kk + 1 < k1 ? s0[1] * a.scale_log2 : -INFINITY;
        const float x2 = kk + 8 < k1 ? s1[0] * a.scale_log2 : -INFINITY;
        const float x3 = kk + 9 < k1 ? s1[1] * a.scale_log2 : -INFINITY;
        const float y0 = kk < k1 ? s0[2] * a.scale_log2 : -INFINITY;
        const float y1 = kk + 1 < k1 ? s0[3] * a.scale_log2 : -INFINITY;
        const float y2 = kk + 8 < k1 ? s1[2] * a.scale_log2 : -INFINITY;
        const float y3 = kk + 9 < k1 ? s1[3] * a.scale_log2 : -INFINITY;
        float mxa = fmaxf(fmaxf(x0, x1), fmaxf(x2, x3));
        float mxb = fmaxf(fmaxf(y0, y1), fmaxf(y2, y3));
        mxa = fmaxf(mxa, __shfl_xor_sync(0xffffffffu, mxa, 1));
        mxa = fmaxf(mxa, __shfl_xor_sync(0xffffffffu, mxa, 2));
        mxb = fmaxf(mxb, __shfl_xor_sync(0xffffffffu, mxb, 1));
        mxb = fmaxf(mxb, __shfl_xor_sync(0xffffffffu, mxb, 2));
        // finite: the first key of every step is in range
        const float mna = fmaxf(m_a, mxa), mnb = fmaxf(m_b, mxb);
        const float alpha_a = exp2f(m_a - mna), alpha_b = exp2f(m_b - mnb);
        m_a = mna;
        m_b = mnb;
        const float p0 = exp2f(x0 - mna), p1 = exp2f(x1 - mna), p2 = exp2f(x2 - mna), p3 = exp2f(x3 - mna);
        const float r0 = exp2f(y0 - mnb), r1 = exp2f(y1 - mnb), r2 = exp2f(y2 - mnb), r3 = exp2f(y3 - mnb);
        l_a = l_a * alpha_a + ((p0 + p1) + (p2 + p3));
        l_b = l_b * alpha_b + ((r0 + r1) + (r2 + r3));
#pragma unroll
        for (int t = 0; t < 16; ++t) {
            o[t][0] *= alpha_a;
            o[t][1] *= alpha_a;
            o[t][2] *= alpha_b;
            o[t][3] *= alpha_b;
        }
        // P as bf16 hi + lo.  Packed rows: rows gid carry P_hi, rows gid+8
        // P_lo of the same head (summed at the end).  Otherwise rows are
        // heads and P_lo is a second mma into the same accumulator.
        const uint32_t ph0 = pack_bf16x2(p0, p1), ph2 = pack_bf16x2(p2, p3);
        const uint32_t pl0 = pack_bf16x2(p0 - bf16lo(ph0), p1 - bf16hi(ph0));
        const uint32_t pl2 = pack_bf16x2(p2 - bf16lo(ph2), p3 - bf16hi(ph2));
        const uint32_t rh0 = pack_bf16x2(r0, r1), rh2 = pack_bf16x2(r2, r3);
        const uint32_t rl0 = pack_bf16x2(r0 - bf16lo(rh0), r1 - bf16hi(rh0));
        const uint32_t rl2 = pack_bf16x2(r2 - bf16lo(rh2), r3 - bf16hi(rh2));
        // ---- O += P V over 16 output tiles (head_dim 16n + t) ----
#pragma unroll
        for (int t = 0; t < 16; ++t) {
            const int h = t >> 3, comp = (t & 7) >> 1;
            const uint32_t sel = (t & 1) ? 0x7632u : 0x5410u;
            const uint32_t wa_ = comp == 0 ? va[h].x : comp == 1 ? va[h].y : comp == 2 ? va[h].z : va[h].w;
            const uint32_t wb_ = comp == 0 ? vb[h].x : comp == 1 ? vb[h].y : comp == 2 ? vb[h].z : vb[h].w;
            const uint32_t wc_ = comp == 0 ? vc2[h].x : comp == 1 ? vc2[h].y : comp == 2 ? vc2[h].z : vc2[h].w;
            const uint32_t wd_ = comp == 0 ? vd[h].x : comp == 1 ? vd[h].y : comp == 2 ? vd[h].z : vd[h].w;
            const uint32_t vb0 = prmt(wa_, wb_, sel), vb1 = prmt(wc_, wd_, sel);
            if constexpr (PACKED) {
                mma_bf16_16816(o[t], ph0, pl0, ph2, pl2, vb0, vb1);
            } else {
                mma_bf16_16816(o[t], ph0, rh0, ph2, rh2, vb0, vb1);
                mma_bf16_16816(o[t], pl0, rl0, pl2, rl2, vb0, vb1);
            }
        }
    };
    // two buffers: the next 16 keys load while the current 16 are processed
    for (int64_t kb = k0; kb < k1; kb += 32) {
        if (kb + 16 < k1) load16(bufB, kb + 16);
        process(bufA, kb);
        if (kb + 16 >= k1) break;
        if (kb + 32 < k1) load16(bufA, kb + 32);
        process(bufB, kb + 16);
    }
    if constexpr (PACKED) {
        // rows gid+8 held the P_lo . V half of the same head
#pragma unroll
        for (int t = 0; t < 16; ++t) {
            o[t][0] += o[t][2];
            o[t][1] += o[t][3];
        }
    }

    // ---- combine the CTA's warps in shared memory (ascending warp order) ----
    l_a += __shfl_xor_sync(0xffffffffu, l_a, 1);
    l_a += __shfl_xor_sync(0xffffffffu, l_a, 2);
    l_b += __shfl_xor_sync(0xffffffffu, l_b, 1);
    l_b += __shfl_xor_sync(0xffffffffu, l_b, 2);
    __shared__ float s_o[kAttnWarps][16][D];   // unnormalised outputs per warp and head
    __shared__ float s_ml[kAttnWarps][16][2];  // (max, sum) per warp and head
    // o[t][0] -> (row gid, dim 32c + t); o[t][1] -> (row gid, dim 32c + 16 + t); [2],[3]: row gid+8
    if (gid < a.g) {
#pragma unroll
        for (int t = 0; t < 16; ++t) {
            s_o[warp][gid][32 * c + t] = o[t][0];
            s_o[warp][gid][32 * c + 16 + t] = o[t][1];
        }
        if (c == 0) {
            s_ml[warp][gid][0] = m_a;
            s_ml[warp][gid][1] = l_a;
        }
    }
    if (!packed_rows && gid + 8 < a.g) {
#pragma unroll
        for (int t = 0; t < 16; ++t) {
            s_o[warp][gid + 8][32 * c + t] = o[t][2];
            s_o[warp][gid + 8][32 * c + 16 + t] = o[t][3];
        }
        if (c == 0) {
            s_ml[warp][gid + 8][0] = m_b;
            s_ml[warp][gid + 8][1] = l_b;
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) TPL_TRACE_AT(2);
    const int dim = threadIdx.x;  // 128 threads, one head_dim column each
    const int cpp_ = cpp;
    const int64_t cbase = ((int64_t)pair * cpp_ + chunk) * a.g;  // this CTA's partial
    for (int hrow = 0; hrow < a.g; ++hrow) {
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kAttnWarps; ++w) M = fmaxf(M, s_ml[w][hrow][0]);
        float num = 0.f, den = 0.f;
#pragma unroll
        for (int w = 0; w < kAttnWarps; ++w) {
            const float mi = s_ml[w][hrow][0];
            const float wt = mi == -INFINITY ? 0.f : exp2f(mi - M);
            num += wt * s_o[w][hrow][dim];
            den += wt * s_ml[w][hrow][1];
        }
        a.part_o[(cbase + hrow) * D + dim] = num;
        if (dim == 0) {
            a.part_ml[(cbase + hrow) * 2 + 0] = M;
            a.part_ml[(cbase + hrow) * 2 + 1] = den;
        }
    }

    // ---- the last CTA of the pair combines the CTA partials in ascending order ----
    __shared__ int s_last;
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        const unsigned prev = atomicAdd(&a.tickets[pair], 1u);
        s_last = prev == (unsigned)(cpp_ - 1);
        if (prev >= (unsigned)cpp_) record_error(2u);
    }
    __syncthreads();
    if (!s_last) {
        if (threadIdx.x == 0) {
            TPL_TRACE_AT(3);
            TPL_TRACE_PUT(TR_ATTN);
        }
        return;
    }
    __threadfence();
    // stage every CTA partial's (max, sum) for this pair
    __shared__ float s_w[64][16];  // weights exp2(m_i - M) per CTA partial and head
    __shared__ float s_M[16], s_den[16], s_new[16];
    __shared__ float s_red[kAttnWarps][16];
    float *s_mlp = &s_o[0][0][0];  // reuse: [cpp][g][2] (cpp <= 64)
    for (int i = threadIdx.x; i < cpp_ * a.g * 2; i += blockDim.x)
        s_mlp[i] = __ldcg(&a.part_ml[(int64_t)pair * cpp_ * a.g * 2 + i]);
    attn_pair_combine<16>(a, pair, cpp_, b, j, dim, lane, warp, s_mlp, s_w, s_M, s_den, s_new, s_red);
    if (threadIdx.x == 0) {
        atomicExch(&a.tickets[pair], 0u);
        TPL_TRACE_AT(3);
        TPL_TRACE_PUT(TR_ATTN);
    }
}


// ---------------------------------------------------------------------------
// Staged variant (query groups of at most 8 heads): the same splits, merge and
// ordered combine, but each warp streams its keys through its own ring of
// kStgStages shared-memory stages of 16 keys (cp.async, 16-byte pieces into
// rows padded to 272 bytes) and reads the mma operands with ldmatrix, so
// four 16-key steps are in flight per warp instead of the two that fit in
// registers.  One CTA per SM; the host gives each (shard, sequence, kv head)
// pair floor(SMs / pairs) CTAs (at least 64 keys per warp), one wave.
//   S: A = q (rows 0-7 hi, rows 8-15 lo of the g heads, standard fragments),
//      B = 8 keys x 16 dims (ldmatrix of K rows);
//   O: A = P (rows 0-7 hi, rows 8-15 lo), B = 16 keys x 8 dims (ldmatrix.trans
//      of V rows); output tile t holds dims 8t + 2c, 8t + 2c + 1.
// ---------------------------------------------------------------------------
constexpr int kStgWarps = kAttnStgWarps;               // two per SM sub-partition
constexpr int kStgStages = 3;
constexpr int kStgRow = 136;                           // padded row, bf16 elements
constexpr int kStgStep = 2 * 16 * kStgRow;             // K and V rows of one stage, elements
constexpr size_t kStgSmem = (size_t)kStgWarps * kStgStages * kStgStep * 2;  // dynamic bytes
static_assert((size_t)kStgWarps * 8 * (128 + 2) * 4 <= kStgSmem, "the warps' merge overlays the rings");
constexpr float kStgLazy = 8.0f;  // the running maximum (log2 units) is raised only past this margin

__global__ void __launch_bounds__(kStgWarps * 32, 1) attn_decode_staged_kernel(const __grid_constant__ AttnArgs a) {
    constexpr int D = 128;
    extern __shared__ __align__(128) __nv_bfloat16 stg_smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gid = lane >> 2, c = lane & 3;
    const int cpp = a.nsplit / kStgWarps;
    const int pair = blockIdx.x / cpp, chunk = blockIdx.x % cpp;
    const int split = chunk * kStgWarps + warp;
    const int jl = pair % a.nkv_s;
    const int sb = pair / a.nkv_s;
    const int b = sb % a.B, s = sb / a.B;
    const int j = s * a.nkv_s + jl;
    const int64_t cache_off = (((int64_t)s * a.batch_cap + b) * a.nkv_s + jl) * a.seq_cap * D;
    const __nv_bfloat16 *Kp = a.kc + cache_off;
    const __nv_bfloat16 *Vp = a.vc + cache_off;
    const int64_t k0 = (int64_t)split * a.kps;
    const int64_t k1 = min(a.keys, k0 + a.kps);
    const int nsteps = k1 > k0 ? (int)((k1 - k0 + 15) / 16) : 0;
    const bool early = a.k_new != nullptr;
    TPL_TRACE_VARS
    if (threadIdx.x == 0) TPL_TRACE_AT(0);
    __nv_bfloat16 *ring = stg_smem + (size_t)warp * kStgStages * kStgStep;

    const uint64_t kvpol = evict_first_policy();  // the cache is read once
    // stage st (keys k0 + 16 st ..) into slot st % kStgStages; keys past k1 read as zero
    auto issue = [&](int st) {
        if (st < nsteps) {
            __nv_bfloat16 *kd = ring + (st % kStgStages) * kStgStep;
            __nv_bfloat16 *vd = kd + 16 * kStgRow;
            const int64_t kb = k0 + 16 * (int64_t)st;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int piece = lane + 32 * i;  // 256 pieces of 16 bytes: 16 rows x 16
                const int r = piece >> 4, col = (piece & 15) * 8;
                const int64_t key = kb + r;
                if (key < k1) {
                    cp_async16_hint(kd + r * kStgRow + col, Kp + key * D + col, kvpol);
                    cp_async16_hint(vd + r * kStgRow + col, Vp + key * D + col, kvpol);
                } else {
                    *reinterpret_cast<uint4 *>(kd + r * kStgRow + col) = make_uint4(0, 0, 0, 0);
                    *reinterpret_cast<uint4 *>(vd + r * kStgRow + col) = make_uint4(0, 0, 0, 0);
                }
            }
        }
        cp_async_commit();  // one group per stage, empty ones included
    };
    if (early)
        for (int st = 0; st < kStgStages - 1; ++st) issue(st);
    pdl_wait();
    pdl_trigger();
    if (threadIdx.x == 0) TPL_TRACE_AT(1);
    if (!early)
        for (int st = 0; st < kStgStages - 1; ++st) issue(st);

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

    // the new token's logits, for whichever CTA of the pair finishes last
    // (the first 128 threads: one head dimension each)
    __shared__ float s_red[kAttnWarps][8];
    const float vnew = warp < kAttnWarps ? attn_new_logits<8>(a, b, j, threadIdx.x, lane, warp, s_red) : 0.f;

    float o[16][4];
#pragma unroll
    for (int t = 0; t < 16; ++t) o[t][0] = o[t][1] = o[t][2] = o[t][3] = 0.f;
    float m_a = -INFINITY, l_a = 0.f;  // head gid: running max (log2 domain), lane-partial sum

    for (int st = 0; st < nsteps; ++st) {
        issue(st + kStgStages - 1);
        asm volatile("cp.async.wait_group %0;" ::"n"(kStgStages - 1) : "memory");
        __syncwarp();
        const __nv_bfloat16 *Ks = ring + (st % kStgStages) * kStgStep;
        const __nv_bfloat16 *Vs = Ks + 16 * kStgRow;
        float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            const int r = (lane & 7) + ((lane >> 4) << 3);
            const int col = 16 * ks + ((lane >> 3) & 1) * 8;
            uint32_t b0, b1, b2, b3;
            ldsm_x4(Ks + r * kStgRow + col, b0, b1, b2, b3);
            mma_bf16_16816(s0, qf[ks][0], qf[ks][1], qf[ks][2], qf[ks][3], b0, b1);
            mma_bf16_16816(s1, qf[ks][0], qf[ks][1], qf[ks][2], qf[ks][3], b2, b3);
        }
        // logits: hi rows + lo rows of the same head; keys kb + 2c, +1 (tile 0), kb + 8 + 2c, +1 (tile 1)
        const int64_t kk = k0 + 16 * (int64_t)st + 2 * c;
        const float x0 = kk < k1 ? (s0[0] + s0[2]) * a.scale_log2 : -INFINITY;
        const float x1 = kk + 1 < k1 ? (s0[1] + s0[3]) * a.scale_log2 : -INFINITY;
        const float x2 = kk + 8 < k1 ? (s1[0] + s1[2]) * a.scale_log2 : -INFINITY;
        const float x3 = kk + 9 < k1 ? (s1[1] + s1[3]) * a.scale_log2 : -INFINITY;
        float mx = fmaxf(fmaxf(x0, x1), fmaxf(x2, x3));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        // mx is finite: the first key of every step is in range.  Raise the
        // running maximum only past the margin; until then p <= 2^kStgLazy.
        if (mx > m_a + kStgLazy) {
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
        const float p0 = exp2f(x0 - m_a), p1 = exp2f(x1 - m_a), p2 = exp2f(x2 - m_a), p3 = exp2f(x3 - m_a);
        l_a += (p0 + p1) + (p2 + p3);
        const uint32_t ph0 = pack_bf16x2(p0, p1), ph2 = pack_bf16x2(p2, p3);
        const uint32_t pl0 = pack_bf16x2(p0 - bf16lo(ph0), p1 - bf16hi(ph0));
        const uint32_t pl2 = pack_bf16x2(p2 - bf16lo(ph2), p3 - bf16hi(ph2));
#pragma unroll
        for (int n2 = 0; n2 < 8; ++n2) {
            const int r = (lane & 7) + (((lane >> 3) & 1) << 3);
            const int col = 16 * n2 + ((lane >> 4) << 3);
            uint32_t v0, v1, v2, v3;
            ldsm_x4_t(Vs + r * kStgRow + col, v0, v1, v2, v3);
            mma_bf16_16816(o[2 * n2], ph0, pl0, ph2, pl2, v0, v1);
            mma_bf16_16816(o[2 * n2 + 1], ph0, pl0, ph2, pl2, v2, v3);
        }
        __syncwarp();  // this slot is refilled by a later issue()
    }
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    if (threadIdx.x == 0) TPL_TRACE_AT(2);
#ifdef TPL_TRACE
    // SM-clock marks of the end (traced builds): every warp's loop done,
    // partial written, arrival counted, combine done
    uint64_t ck[4] = {0, 0, 0, 0};
#endif
    // rows gid + 8 held the P_lo . V half of the same head
#pragma unroll
    for (int t = 0; t < 16; ++t) {
        o[t][0] += o[t][2];
        o[t][1] += o[t][3];
    }
    l_a += __shfl_xor_sync(0xffffffffu, l_a, 1);
    l_a += __shfl_xor_sync(0xffffffffu, l_a, 2);

    // ---- merge the CTA's warps (ascending warp order), then the CTA partials.
    //      The warps' outputs go to the (now idle) stage rings ----
    __syncthreads();  // every warp is done with its ring
    float(*s_o)[8][D] = reinterpret_cast<float(*)[8][D]>(stg_smem);                       // [kStgWarps][8][D]
    float(*s_ml)[8][2] = reinterpret_cast<float(*)[8][2]>(stg_smem + kStgWarps * 8 * D * 2);  // [kStgWarps][8][2]
    if (gid < a.g) {
#pragma unroll
        for (int t = 0; t < 16; ++t) {
            s_o[warp][gid][8 * t + 2 * c] = o[t][0];
            s_o[warp][gid][8 * t + 2 * c + 1] = o[t][1];
        }
        if (c == 0) {
            s_ml[warp][gid][0] = m_a;
            s_ml[warp][gid][1] = l_a;
        }
    }
    __syncthreads();
#ifdef TPL_TRACE
    if (threadIdx.x == 0) ck[0] = (uint64_t)clock64();
#endif
    // thread t: head dimension t % 128 of the heads t / 128, + 2, + 4, ...
    const int dim = threadIdx.x & (D - 1);
    const int64_t cbase = ((int64_t)pair * cpp + chunk) * a.g;
    for (int hrow = threadIdx.x / D; hrow < a.g; hrow += kStgWarps * 32 / D) {
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kStgWarps; ++w) M = fmaxf(M, s_ml[w][hrow][0]);
        float num = 0.f, den = 0.f;
#pragma unroll
        for (int w = 0; w < kStgWarps; ++w) {
            const float mi = s_ml[w][hrow][0];
            const float wt = mi == -INFINITY ? 0.f : exp2f(mi - M);
            num += wt * s_o[w][hrow][dim];
            den += wt * s_ml[w][hrow][1];
        }
        a.part_o[(cbase + hrow) * D + dim] = num;
        if (dim == 0) {
            a.part_ml[(cbase + hrow) * 2 + 0] = M;
            a.part_ml[(cbase + hrow) * 2 + 1] = den;
        }
    }
    __shared__ int s_last;
    __threadfence();
    __syncthreads();
#ifdef TPL_TRACE
    if (threadIdx.x == 0) ck[1] = (uint64_t)clock64();
#endif
    if (threadIdx.x == 0) {
        const unsigned prev = atomicAdd(&a.tickets[pair], 1u);
        s_last = prev == (unsigned)(cpp - 1);
        if (prev >= (unsigned)cpp) record_error(2u);
    }
    __syncthreads();
#ifdef TPL_TRACE
    if (threadIdx.x == 0) ck[2] = ck[3] = (uint64_t)clock64();
#endif
    if (!s_last) {
        if (threadIdx.x == 0) {
            TPL_TRACE_AT(3);
            TPL_TRACE_PUT(TR_ATTN);
#ifdef TPL_TRACE
            trace_put(202, ck);
#endif
        }
        return;
    }
    __threadfence();
    // the pair's combine runs on the first 128 threads (one head dimension each)
    if (warp >= kAttnWarps) return;
    __shared__ float s_w[kAttnMaxCtasPerPair][8];
    __shared__ float s_M[8], s_den[8], s_new[8];
    __shared__ float s_mlp[kAttnMaxCtasPerPair * 8 * 2];
    for (int i = threadIdx.x; i < cpp * a.g * 2; i += kAttnWarps * 32)
        s_mlp[i] = __ldcg(&a.part_ml[(int64_t)pair * cpp * a.g * 2 + i]);
    attn_pair_combine<8>(a, pair, cpp, b, j, dim, lane, warp, s_mlp, s_w, s_M, s_den, s_new, s_red, true, vnew);
    if (threadIdx.x == 0) {
        atomicExch(&a.tickets[pair], 0u);
        TPL_TRACE_AT(3);
        TPL_TRACE_PUT(TR_ATTN);
#ifdef TPL_TRACE
        ck[3] = (uint64_t)clock64();
        trace_put(212, ck);
#endif
    }
}

}  // namespace tpl
