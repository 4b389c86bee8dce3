// Causal GQA attention of a prefill chunk ("Tensor parallel scaling curves",
// "Prefill vs decode: different curves"; each shard attends over its own heads, "What
// tensor parallelism actually splits"): token i attends keys 0..i of the
// chunk.  One CTA per (kv head, 16-token row tile, chunk of the head's query
// group); warp w handles one query head of the chunk for those 16 tokens, so
// the K/V tiles staged in shared memory serve every head of the chunk.  CTAs
// start with the longest rows (the causal triangle's heavy end).
//
// Precision: q, k, v, P are each carried as bf16 hi + lo; Q K^T is
// q_hi.k_hi + q_hi.k_lo + q_lo.k_hi and P V is P_hi.v_hi + P_hi.v_lo +
// P_lo.v_hi (mma.sync m16n8k16, fp32 accumulate), about 16 mantissa bits.
// K/V tiles of 64 keys are double-buffered with cp.async; ldmatrix reads the
// B operands (transposed for V) from rows padded to 272 bytes.
#pragma once

#include "tpl_common.cuh"
#include "tpl_internal.h"

namespace tpl {

constexpr int kApKeys = 64;              // keys per staged tile
constexpr int kApRow = 136;              // padded row (bf16 elements): 272 bytes
constexpr int kApTile = kApKeys * kApRow;  // elements per plane
constexpr int kApMaxWarps = 8;
constexpr size_t kApSmem = (size_t)2 * 4 * kApTile * 2;  // two buffers of four planes

struct AttnPrefillArgs {
    const float *q32;                 // [T][nq][128]
    const __nv_bfloat16 *khi, *vhi;   // cache planes, shard-major [t][batch_cap][nkv_s][seq_cap][128] (batch row 0)
    const __nv_bfloat16 *klo, *vlo;   // [T][nkv][128] low parts
    int64_t seq_cap;
    int batch_cap;
    int T, nq, nkv, nkv_s, g;
    int p0;                           // position of the chunk's first token (cache slots below hold earlier keys)
    int gc, wpc;                      // chunks per query group, heads (warps) per chunk
    float scale_log2;
    __nv_bfloat16 *o_hi, *o_lo;       // [T][nq*128]: output as bf16 hi + lo (the O projection's split operand)
};

__global__ void __launch_bounds__(kApMaxWarps * 32) attn_prefill_kernel(const __grid_constant__ AttnPrefillArgs a) {
    constexpr int D = 128;
    extern __shared__ __align__(128) __nv_bfloat16 apsm[];  // [2 buffers][4 planes: khi, klo, vhi, vlo][64][136]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, gid = lane >> 2, c = lane & 3;
    const int nthreads = blockDim.x;
    const int ntile = (a.T + 15) / 16;
    const int per_rt = a.nkv * a.gc;
    const int rt = ntile - 1 - (int)(blockIdx.x / per_rt);  // row tile, longest first
    const int rem = (int)(blockIdx.x % per_rt);
    const int j = rem / a.gc, chunk = rem % a.gc;           // global kv head, group chunk
    const int s = j / a.nkv_s, jl = j % a.nkv_s;
    const int head = j * a.g + chunk * a.wpc + warp;
    const int t0 = rt * 16;
    const int t_last = min(a.T - 1, t0 + 15);
    const int nkb = (a.p0 + t_last) / kApKeys + 1;  // key tiles up to the last token's
    const int64_t cache_off = (((int64_t)s * a.batch_cap) * a.nkv_s + jl) * a.seq_cap * D;

    pdl_wait();
    pdl_trigger();

    auto stage = [&](int kb, int buf) {
        __nv_bfloat16 *base = apsm + (size_t)buf * 4 * kApTile;
        // 64 keys x 128 dims x 4 planes in 16-byte pieces (16 per row)
        for (int u = threadIdx.x; u < 4 * kApKeys * 16; u += nthreads) {
            const int plane = u / (kApKeys * 16), r = (u / 16) % kApKeys, piece = u % 16;
            const int key = kb * kApKeys + r;
            __nv_bfloat16 *dst = base + (size_t)plane * kApTile + r * kApRow + piece * 8;
            // keys below p0 come from earlier chunks: exact in bf16, no low part
            if (key < a.p0 + a.T && ((plane & 1) == 0 || key >= a.p0)) {
                const __nv_bfloat16 *src;
                if (plane == 0) src = a.khi + cache_off + (int64_t)key * D;
                else if (plane == 1) src = a.klo + ((int64_t)(key - a.p0) * a.nkv + j) * D;
                else if (plane == 2) src = a.vhi + cache_off + (int64_t)key * D;
                else src = a.vlo + ((int64_t)(key - a.p0) * a.nkv + j) * D;
                cp_async16(dst, src + piece * 8);
            } else {
                *reinterpret_cast<uint4 *>(dst) = make_uint4(0, 0, 0, 0);
            }
        }
    };

    // Q fragments (rows = tokens t0 + gid, t0 + gid + 8), hi and lo
    uint32_t qh[8][4], ql[8][4];
    {
        const int ta = t0 + gid, tb = t0 + gid + 8;
        for (int ks = 0; ks < 8; ++ks) {
            float va[4] = {0.f, 0.f, 0.f, 0.f}, vb[4] = {0.f, 0.f, 0.f, 0.f};  // (k 2c,2c+1), (k 2c+8, +9)
            if (ta < a.T) {
                const float *p = a.q32 + ((int64_t)ta * a.nq + head) * D + 16 * ks + 2 * c;
                const float2 x0 = *reinterpret_cast<const float2 *>(p), x1 = *reinterpret_cast<const float2 *>(p + 8);
                va[0] = x0.x; va[1] = x0.y; va[2] = x1.x; va[3] = x1.y;
            }
            if (tb < a.T) {
                const float *p = a.q32 + ((int64_t)tb * a.nq + head) * D + 16 * ks + 2 * c;
                const float2 x0 = *reinterpret_cast<const float2 *>(p), x1 = *reinterpret_cast<const float2 *>(p + 8);
                vb[0] = x0.x; vb[1] = x0.y; vb[2] = x1.x; vb[3] = x1.y;
            }
            // a0a1: row gid k 2c; a2a3: row gid+8 k 2c; a4a5: row gid k 2c+8; a6a7: row gid+8 k 2c+8
            const uint32_t h0 = pack_bf16x2(va[0], va[1]), h1 = pack_bf16x2(vb[0], vb[1]);
            const uint32_t h2 = pack_bf16x2(va[2], va[3]), h3 = pack_bf16x2(vb[2], vb[3]);
            qh[ks][0] = h0; qh[ks][1] = h1; qh[ks][2] = h2; qh[ks][3] = h3;
            ql[ks][0] = pack_bf16x2(va[0] - bf16lo(h0), va[1] - bf16hi(h0));
            ql[ks][1] = pack_bf16x2(vb[0] - bf16lo(h1), vb[1] - bf16hi(h1));
            ql[ks][2] = pack_bf16x2(va[2] - bf16lo(h2), va[3] - bf16hi(h2));
            ql[ks][3] = pack_bf16x2(vb[2] - bf16lo(h3), vb[3] - bf16hi(h3));
        }
    }

    float o[16][4];
#pragma unroll
    for (int t = 0; t < 16; ++t) o[t][0] = o[t][1] = o[t][2] = o[t][3] = 0.f;
    float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.f, l_b = 0.f;
    const int ra = t0 + gid, rb_ = t0 + gid + 8;  // query tokens of rows gid, gid+8
    const int pa = a.p0 + ra, pb = a.p0 + rb_;    // and their positions

    stage(0, 0);
    cp_async_commit();
    for (int kb = 0; kb < nkb; ++kb) {
        const int buf = kb & 1;
        if (kb + 1 < nkb) {
            stage(kb + 1, buf ^ 1);
            cp_async_commit();
            cp_async_wait_1();
        } else {
            cp_async_wait_0();
        }
        __syncthreads();
        const __nv_bfloat16 *Kh = apsm + (size_t)buf * 4 * kApTile;
        const __nv_bfloat16 *Kl = Kh + kApTile, *Vh = Kh + 2 * kApTile, *Vl = Kh + 3 * kApTile;
        // 4 sub-blocks of 16 keys
        for (int sb = 0; sb < kApKeys / 16; ++sb) {
            const int key0 = kb * kApKeys + sb * 16;
            if (key0 > a.p0 + t_last) break;
            float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};  // keys key0+.. tile0 / tile1
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                // B fragments of K^T for keys key0..+15, d 16ks..+15 (ldmatrix x4 -> two n-tiles)
                const int r = sb * 16 + (lane & 7) + ((lane >> 4) << 3);
                const int col = 16 * ks + ((lane >> 3) & 1) * 8;
                uint32_t bh0, bh1, bh2, bh3, bl0, bl1, bl2, bl3;
                ldsm_x4(Kh + r * kApRow + col, bh0, bh1, bh2, bh3);
                ldsm_x4(Kl + r * kApRow + col, bl0, bl1, bl2, bl3);
                // tile0: (bh0, bh1); tile1: (bh2, bh3)
                mma_bf16_16816(s0, qh[ks][0], qh[ks][1], qh[ks][2], qh[ks][3], bh0, bh1);
                mma_bf16_16816(s0, qh[ks][0], qh[ks][1], qh[ks][2], qh[ks][3], bl0, bl1);
                mma_bf16_16816(s0, ql[ks][0], ql[ks][1], ql[ks][2], ql[ks][3], bh0, bh1);
                mma_bf16_16816(s1, qh[ks][0], qh[ks][1], qh[ks][2], qh[ks][3], bh2, bh3);
                mma_bf16_16816(s1, qh[ks][0], qh[ks][1], qh[ks][2], qh[ks][3], bl2, bl3);
                mma_bf16_16816(s1, ql[ks][0], ql[ks][1], ql[ks][2], ql[ks][3], bh2, bh3);
            }
            // causal mask and online softmax; s0 cols = keys key0+2c, +1; s1 = key0+8+2c, +1
            const int kk = key0 + 2 * c;
            const float x0 = kk <= pa ? s0[0] * a.scale_log2 : -INFINITY;
            const float x1 = kk + 1 <= pa ? s0[1] * a.scale_log2 : -INFINITY;
            const float x2 = kk + 8 <= pa ? s1[0] * a.scale_log2 : -INFINITY;
            const float x3 = kk + 9 <= pa ? s1[1] * a.scale_log2 : -INFINITY;
            const float y0 = kk <= pb ? s0[2] * a.scale_log2 : -INFINITY;
            const float y1 = kk + 1 <= pb ? s0[3] * a.scale_log2 : -INFINITY;
            const float y2 = kk + 8 <= pb ? s1[2] * a.scale_log2 : -INFINITY;
            const float y3 = kk + 9 <= pb ? s1[3] * a.scale_log2 : -INFINITY;
            float mxa = fmaxf(fmaxf(x0, x1), fmaxf(x2, x3));
            float mxb = fmaxf(fmaxf(y0, y1), fmaxf(y2, y3));
            mxa = fmaxf(mxa, __shfl_xor_sync(0xffffffffu, mxa, 1));
            mxa = fmaxf(mxa, __shfl_xor_sync(0xffffffffu, mxa, 2));
            mxb = fmaxf(mxb, __shfl_xor_sync(0xffffffffu, mxb, 1));
            mxb = fmaxf(mxb, __shfl_xor_sync(0xffffffffu, mxb, 2));
            const float mna = fmaxf(m_a, mxa), mnb = fmaxf(m_b, mxb);
            // a row whose keys are all masked so far keeps max -inf: use 0 as the base
            const float ba = mna == -INFINITY ? 0.f : mna, bb = mnb == -INFINITY ? 0.f : mnb;
            const float al_a = exp2f(m_a - ba), al_b = exp2f(m_b - bb);
            m_a = mna;
            m_b = mnb;
            const float p0 = exp2f(x0 - ba), p1 = exp2f(x1 - ba), p2 = exp2f(x2 - ba), p3 = exp2f(x3 - ba);
            const float r0 = exp2f(y0 - bb), r1 = exp2f(y1 - bb), r2 = exp2f(y2 - bb), r3 = exp2f(y3 - bb);
            l_a = l_a * al_a + ((p0 + p1) + (p2 + p3));
            l_b = l_b * al_b + ((r0 + r1) + (r2 + r3));
#pragma unroll
            for (int t = 0; t < 16; ++t) {
                o[t][0] *= al_a;
                o[t][1] *= al_a;
                o[t][2] *= al_b;
                o[t][3] *= al_b;
            }
            const uint32_t ph0 = pack_bf16x2(p0, p1), ph1 = pack_bf16x2(r0, r1);
            const uint32_t ph2 = pack_bf16x2(p2, p3), ph3 = pack_bf16x2(r2, r3);
            const uint32_t pl0 = pack_bf16x2(p0 - bf16lo(ph0), p1 - bf16hi(ph0));
            const uint32_t pl1 = pack_bf16x2(r0 - bf16lo(ph1), r1 - bf16hi(ph1));
            const uint32_t pl2 = pack_bf16x2(p2 - bf16lo(ph2), p3 - bf16hi(ph2));
            const uint32_t pl3 = pack_bf16x2(r2 - bf16lo(ph3), r3 - bf16hi(ph3));
            // P V: B fragments of V (keys key0..+15, d 16n..+15) with ldmatrix.trans
#pragma unroll
            for (int n2 = 0; n2 < 8; ++n2) {
                const int r = sb * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
                const int col = 16 * n2 + ((lane >> 4) << 3);
                uint32_t vh0, vh1, vh2, vh3, vl0, vl1, vl2, vl3;
                ldsm_x4_t(Vh + r * kApRow + col, vh0, vh1, vh2, vh3);
                ldsm_x4_t(Vl + r * kApRow + col, vl0, vl1, vl2, vl3);
                // n-tile 2*n2: (vh0, vh1); n-tile 2*n2+1: (vh2, vh3)
                mma_bf16_16816(o[2 * n2], ph0, ph1, ph2, ph3, vh0, vh1);
                mma_bf16_16816(o[2 * n2], ph0, ph1, ph2, ph3, vl0, vl1);
                mma_bf16_16816(o[2 * n2], pl0, pl1, pl2, pl3, vh0, vh1);
                mma_bf16_16816(o[2 * n2 + 1], ph0, ph1, ph2, ph3, vh2, vh3);
                mma_bf16_16816(o[2 * n2 + 1], ph0, ph1, ph2, ph3, vl2, vl3);
                mma_bf16_16816(o[2 * n2 + 1], pl0, pl1, pl2, pl3, vh2, vh3);
            }
        }
        __syncthreads();  // the buffer is restaged two tiles later
    }
    l_a += __shfl_xor_sync(0xffffffffu, l_a, 1);
    l_a += __shfl_xor_sync(0xffffffffu, l_a, 2);
    l_b += __shfl_xor_sync(0xffffffffu, l_b, 1);
    l_b += __shfl_xor_sync(0xffffffffu, l_b, 2);
    // o[t]: c0,c1 = (row gid, d 8t + 2c, +1), c2,c3 = row gid+8
    const float ia = 1.0f / l_a, ib = 1.0f / l_b;
#pragma unroll
    for (int t = 0; t < 16; ++t) {
        const int dcol = 8 * t + 2 * c;
        if (ra < a.T) {
            const int64_t base = (int64_t)ra * a.nq * D + (int64_t)head * D + dcol;
            const float v0 = o[t][0] * ia, v1 = o[t][1] * ia;
            const uint32_t h = pack_bf16x2(v0, v1);
            *reinterpret_cast<uint32_t *>(a.o_hi + base) = h;
            *reinterpret_cast<uint32_t *>(a.o_lo + base) = pack_bf16x2(v0 - bf16lo(h), v1 - bf16hi(h));
        }
        if (rb_ < a.T) {
            const int64_t base = (int64_t)rb_ * a.nq * D + (int64_t)head * D + dcol;
            const float v0 = o[t][2] * ib, v1 = o[t][3] * ib;
            const uint32_t h = pack_bf16x2(v0, v1);
            *reinterpret_cast<uint32_t *>(a.o_hi + base) = h;
            *reinterpret_cast<uint32_t *>(a.o_lo + base) = pack_bf16x2(v0 - bf16lo(h), v1 - bf16hi(h));
        }
    }
}

}  // namespace tpl
