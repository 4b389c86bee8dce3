// Owned-head GQA decode attention ("Tensor parallel scaling curves", "What
// tensor parallelism actually splits": attention runs on the heads a shard
// owns, with no exchange).  One (shard, sequence, kv head) pair is split over
// its S+1 keys into `nsplit` ranges; each warp handles one range with an
// online softmax and writes (max, sum, unnormalised output); the last CTA of
// the pair to arrive (an arrival counter, no waiting) combines the ranges in
// ascending order.
//
// Per warp, 16 keys per step on the tensor cores (mma.sync m16n8k16, bf16):
//   S = Q K^T  -- A = the g query heads of the kv head (rows, zero-padded to
//                 16), B = 8 keys; the head_dim index of each 16-wide step is
//                 permuted so that a lane's K operands are the 64 contiguous
//                 bytes K[key][32m + 8c .. +8), m = 0..3;
//   O += P V   -- A = P from the S accumulators (register reuse), B = V with
//                 output column n of tile t mapped to head_dim 16n + t, so a
//                 lane's V operands are 32 contiguous bytes per key.
// K and V are streamed straight from HBM with 16-byte loads.
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
    int64_t keys;  // S + 1
    int nsplit, kps;
    float scale_log2;  // log2(e) / sqrt(head_dim)
    float *part_o;     // [pairs][nsplit][g][128]
    float *part_ml;    // [pairs][nsplit][g][2]
    unsigned *tickets; // [pairs]
    void *o;           // [B][nq*128] activation type
    int o_f32;
};

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

    pdl_wait();
    pdl_trigger();

    // Q fragments: rows gid (and gid+8) = query heads j*g + row, bf16.
    uint32_t qa[16], qb[16];  // [m*4 + {0..3}]: bf16x2 of q cols 32m+8c+{0,1},{2,3},{4,5},{6,7}
#pragma unroll
    for (int i = 0; i < 16; ++i) { qa[i] = 0u; qb[i] = 0u; }
    if (gid < a.g) {
        const float *qp = a.q + ((int64_t)b * a.nq + (int64_t)j * a.g + gid) * D;
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            const float4 x0 = *reinterpret_cast<const float4 *>(qp + 32 * m + 8 * c);
            const float4 x1 = *reinterpret_cast<const float4 *>(qp + 32 * m + 8 * c + 4);
            qa[m * 4 + 0] = pack_bf16x2(x0.x, x0.y);
            qa[m * 4 + 1] = pack_bf16x2(x0.z, x0.w);
            qa[m * 4 + 2] = pack_bf16x2(x1.x, x1.y);
            qa[m * 4 + 3] = pack_bf16x2(x1.z, x1.w);
        }
    }
    if (gid + 8 < a.g) {
        const float *qp = a.q + ((int64_t)b * a.nq + (int64_t)j * a.g + gid + 8) * D;
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            const float4 x0 = *reinterpret_cast<const float4 *>(qp + 32 * m + 8 * c);
            const float4 x1 = *reinterpret_cast<const float4 *>(qp + 32 * m + 8 * c + 4);
            qb[m * 4 + 0] = pack_bf16x2(x0.x, x0.y);
            qb[m * 4 + 1] = pack_bf16x2(x0.z, x0.w);
            qb[m * 4 + 2] = pack_bf16x2(x1.x, x1.y);
            qb[m * 4 + 3] = pack_bf16x2(x1.z, x1.w);
        }
    }

    float o[16][4];
#pragma unroll
    for (int t = 0; t < 16; ++t) o[t][0] = o[t][1] = o[t][2] = o[t][3] = 0.f;
    float m_a = -INFINITY, m_b = -INFINITY;  // running max of rows gid, gid+8 (log2 domain)
    float l_a = 0.f, l_b = 0.f;              // lane-partial running sums

    for (int64_t kb = k0; kb < k1; kb += 16) {
        // ---- K operands: keys kb+gid (tile 0) and kb+8+gid (tile 1) ----
        uint4 kt0[4], kt1[4];
        {
            const int64_t key0 = kb + gid, key1 = kb + 8 + gid;
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                kt0[m] = key0 < k1 ? ldg_stream(Kp + key0 * D + 32 * m + 8 * c) : make_uint4(0, 0, 0, 0);
                kt1[m] = key1 < k1 ? ldg_stream(Kp + key1 * D + 32 * m + 8 * c) : make_uint4(0, 0, 0, 0);
            }
        }
        // ---- V operands: keys kb+2c, kb+2c+1, kb+8+2c, kb+9+2c; head_dim 16*gid .. +16 ----
        uint4 va[2], vb[2], vc2[2], vd[2];
        {
            const int64_t ka = kb + 2 * c, kbb = ka + 1, kc_ = ka + 8, kd = ka + 9;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int col = 16 * gid + 8 * h;
                va[h] = ka < k1 ? ldg_stream(Vp + ka * D + col) : make_uint4(0, 0, 0, 0);
                vb[h] = kbb < k1 ? ldg_stream(Vp + kbb * D + col) : make_uint4(0, 0, 0, 0);
                vc2[h] = kc_ < k1 ? ldg_stream(Vp + kc_ * D + col) : make_uint4(0, 0, 0, 0);
                vd[h] = kd < k1 ? ldg_stream(Vp + kd * D + col) : make_uint4(0, 0, 0, 0);
            }
        }
        // ---- scores ----
        float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            mma_bf16_16816(s0, qa[m * 4 + 0], qb[m * 4 + 0], qa[m * 4 + 1], qb[m * 4 + 1], kt0[m].x, kt0[m].y);
            mma_bf16_16816(s0, qa[m * 4 + 2], qb[m * 4 + 2], qa[m * 4 + 3], qb[m * 4 + 3], kt0[m].z, kt0[m].w);
            mma_bf16_16816(s1, qa[m * 4 + 0], qb[m * 4 + 0], qa[m * 4 + 1], qb[m * 4 + 1], kt1[m].x, kt1[m].y);
            mma_bf16_16816(s1, qa[m * 4 + 2], qb[m * 4 + 2], qa[m * 4 + 3], qb[m * 4 + 3], kt1[m].z, kt1[m].w);
        }
        // s0: [row gid][keys kb+2c, +1], [row gid+8][...]; s1: keys kb+8+2c, +1
        const int64_t kk = kb + 2 * c;
        float x0 = kk < k1 ? s0[0] * a.scale_log2 : -INFINITY;
        float x1 = kk + 1 < k1 ? s0[1] * a.scale_log2 : -INFINITY;
        float x2 = kk + 8 < k1 ? s1[0] * a.scale_log2 : -INFINITY;
        float x3 = kk + 9 < k1 ? s1[1] * a.scale_log2 : -INFINITY;
        float y0 = kk < k1 ? s0[2] * a.scale_log2 : -INFINITY;
        float y1 = kk + 1 < k1 ? s0[3] * a.scale_log2 : -INFINITY;
        float y2 = kk + 8 < k1 ? s1[2] * a.scale_log2 : -INFINITY;
        float y3 = kk + 9 < k1 ? s1[3] * a.scale_log2 : -INFINITY;
        float mxa = fmaxf(fmaxf(x0, x1), fmaxf(x2, x3));
        float mxb = fmaxf(fmaxf(y0, y1), fmaxf(y2, y3));
        mxa = fmaxf(mxa, __shfl_xor_sync(0xffffffffu, mxa, 1));
        mxa = fmaxf(mxa, __shfl_xor_sync(0xffffffffu, mxa, 2));
        mxb = fmaxf(mxb, __shfl_xor_sync(0xffffffffu, mxb, 1));
        mxb = fmaxf(mxb, __shfl_xor_sync(0xffffffffu, mxb, 2));
        const float mna = fmaxf(m_a, mxa), mnb = fmaxf(m_b, mxb);
        // mna is finite: the first key of every step is in range
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
        const uint32_t pa0 = pack_bf16x2(p0, p1), pa1 = pack_bf16x2(r0, r1);
        const uint32_t pa2 = pack_bf16x2(p2, p3), pa3 = pack_bf16x2(r2, r3);
        // ---- O += P V over 16 output tiles (head_dim 16n + t) ----
#pragma unroll
        for (int t = 0; t < 16; ++t) {
            const int h = t >> 3, comp = (t & 7) >> 1;
            const uint32_t sel = (t & 1) ? 0x7632u : 0x5410u;
            const uint32_t wa_ = comp == 0 ? va[h].x : comp == 1 ? va[h].y : comp == 2 ? va[h].z : va[h].w;
            const uint32_t wb_ = comp == 0 ? vb[h].x : comp == 1 ? vb[h].y : comp == 2 ? vb[h].z : vb[h].w;
            const uint32_t wc_ = comp == 0 ? vc2[h].x : comp == 1 ? vc2[h].y : comp == 2 ? vc2[h].z : vc2[h].w;
            const uint32_t wd_ = comp == 0 ? vd[h].x : comp == 1 ? vd[h].y : comp == 2 ? vd[h].z : vd[h].w;
            mma_bf16_16816(o[t], pa0, pa1, pa2, pa3, prmt(wa_, wb_, sel), prmt(wc_, wd_, sel));
        }
    }

    // ---- write this split's partial result ----
    l_a += __shfl_xor_sync(0xffffffffu, l_a, 1);
    l_a += __shfl_xor_sync(0xffffffffu, l_a, 2);
    l_b += __shfl_xor_sync(0xffffffffu, l_b, 1);
    l_b += __shfl_xor_sync(0xffffffffu, l_b, 2);
    const int64_t pbase = ((int64_t)pair * a.nsplit + split) * a.g;
    // o[t][0] -> (row gid, dim 32c + t); o[t][1] -> (row gid, dim 32c + 16 + t); [2],[3]: row gid+8
    if (gid < a.g) {
        float *dst = a.part_o + (pbase + gid) * D + 32 * c;
#pragma unroll
        for (int t = 0; t < 16; t += 4) {
            *reinterpret_cast<float4 *>(dst + t) = make_float4(o[t][0], o[t + 1][0], o[t + 2][0], o[t + 3][0]);
            *reinterpret_cast<float4 *>(dst + 16 + t) = make_float4(o[t][1], o[t + 1][1], o[t + 2][1], o[t + 3][1]);
        }
        if (c == 0) {
            a.part_ml[(pbase + gid) * 2 + 0] = m_a;
            a.part_ml[(pbase + gid) * 2 + 1] = l_a;
        }
    }
    if (gid + 8 < a.g) {
        float *dst = a.part_o + (pbase + gid + 8) * D + 32 * c;
#pragma unroll
        for (int t = 0; t < 16; t += 4) {
            *reinterpret_cast<float4 *>(dst + t) = make_float4(o[t][2], o[t + 1][2], o[t + 2][2], o[t + 3][2]);
            *reinterpret_cast<float4 *>(dst + 16 + t) = make_float4(o[t][3], o[t + 1][3], o[t + 2][3], o[t + 3][3]);
        }
        if (c == 0) {
            a.part_ml[(pbase + gid + 8) * 2 + 0] = m_b;
            a.part_ml[(pbase + gid + 8) * 2 + 1] = l_b;
        }
    }

    // ---- the last CTA of the pair combines all splits in ascending order ----
    __shared__ int s_last;
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        const unsigned prev = atomicAdd(&a.tickets[pair], 1u);
        s_last = prev == (unsigned)(cpp - 1);
        if (prev >= (unsigned)cpp) record_error(2u);
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    const int dim = threadIdx.x;  // 128 threads, one head_dim column each
    for (int hrow = 0; hrow < a.g; ++hrow) {
        float M = -INFINITY;
        for (int sp = 0; sp < a.nsplit; ++sp)
            M = fmaxf(M, __ldcg(&a.part_ml[(((int64_t)pair * a.nsplit + sp) * a.g + hrow) * 2]));
        float num = 0.f, den = 0.f;
        for (int sp = 0; sp < a.nsplit; ++sp) {
            const int64_t pb = ((int64_t)pair * a.nsplit + sp) * a.g + hrow;
            const float mi = __ldcg(&a.part_ml[pb * 2]);
            const float w = mi == -INFINITY ? 0.f : exp2f(mi - M);
            num += w * __ldcg(&a.part_o[pb * D + dim]);
            den += w * __ldcg(&a.part_ml[pb * 2 + 1]);
        }
        store_act(a.o, a.o_f32, ((int64_t)b * a.nq + (int64_t)j * a.g + hrow) * D + dim, num / den);
    }
    if (threadIdx.x == 0) atomicExch(&a.tickets[pair], 0u);
}

}  // namespace tpl
