// Rotary position embedding of one decode step (TPL_ROPE): q [B][n_q][128]
// and the new keys k_new [B][n_kv][128] (fp32, written by the QKV projection)
// are turned in place to position `pos`, and the rotated key, rounded to
// bf16, replaces the unrotated one in cache slot `pos`.  For e < 64 the pair
// (v[e], v[e + 64]) is rotated by pos * theta[e] (RoFormer's rotation in the
// half-split pairing).  One thread per (token, head, pair): 64 threads of a
// warp pair cover one head; values are touched once, so the kernel is a
// short memory pass.
#pragma once

#include <cuda_bf16.h>

#include "tpl_common.cuh"

namespace tpl {

struct RopeArgs {
    float *q, *knew;
    __nv_bfloat16 *kc;  // shard-major cache [t][batch_cap][nkv_s][seq_cap][128]
    int B, nq, nkv, nkv_s, batch_cap;
    int64_t seq_cap, pos;
    double theta[64];
};

constexpr int kRopeThreads = 256;  // 4 heads per block

__global__ void __launch_bounds__(kRopeThreads) rope_decode_kernel(const __grid_constant__ RopeArgs a) {
    pdl_wait();
    pdl_trigger();
    const int e = threadIdx.x & 63;
    const int64_t head_all = (int64_t)blockIdx.x * (kRopeThreads / 64) + (threadIdx.x >> 6);
    const int heads = a.nq + a.nkv;
    if (head_all >= (int64_t)a.B * heads) return;
    const int b = (int)(head_all / heads), h = (int)(head_all % heads);
    float c, s;
    rope_cs((double)a.pos, a.theta[e], c, s);
    float *v = h < a.nq ? a.q + ((int64_t)b * a.nq + h) * 128 : a.knew + ((int64_t)b * a.nkv + (h - a.nq)) * 128;
    const float x0 = v[e], x1 = v[e + 64];
    const float r0 = x0 * c - x1 * s, r1 = x1 * c + x0 * s;
    v[e] = r0;
    v[e + 64] = r1;
    if (h >= a.nq) {
        const int j = h - a.nq, sh = j / a.nkv_s, jl = j % a.nkv_s;
        __nv_bfloat16 *dst = a.kc + ((((int64_t)sh * a.batch_cap + b) * a.nkv_s + jl) * a.seq_cap + a.pos) * 128;
        dst[e] = __float2bfloat16_rn(r0);
        dst[e + 64] = __float2bfloat16_rn(r1);
    }
}

}  // namespace tpl
