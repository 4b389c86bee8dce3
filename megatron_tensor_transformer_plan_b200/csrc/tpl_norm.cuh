// RMSNorm with the result split into bf16 hi + lo planes: the operand the
// tensor-core projections multiply twice against the bf16 weights.
#pragma once

#include "tpl_common.cuh"

namespace tpl {

// a = x * gamma / sqrt(mean(x^2) + eps) (or a = x without TPL_NORM), split
// into bf16 hi = rn(a) and lo = rn(a - hi).  One CTA per token row; CTAs at
// rows >= rows_valid write zero rows (padding of a fixed-height operand).
__global__ void __launch_bounds__(256) norm_split_kernel(const void *x, int x_f32, const float *gamma, float eps,
                                                         int norm, int H, __nv_bfloat16 *hi, __nv_bfloat16 *lo,
                                                         int rows_valid) {
    __shared__ float s_red[8];
    pdl_wait();
    pdl_trigger();
    const int64_t row = blockIdx.x;
    const int n8 = H / 8;
    if (row >= rows_valid) {
        for (int c = threadIdx.x; c < n8; c += blockDim.x) {
            *reinterpret_cast<uint4 *>(hi + row * H + 8 * c) = make_uint4(0, 0, 0, 0);
            *reinterpret_cast<uint4 *>(lo + row * H + 8 * c) = make_uint4(0, 0, 0, 0);
        }
        return;
    }
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

// The decode projections' operand without the RMSNorm factor: rows 0..B-1 of
// x * gamma (gamma NULL: x) as bf16 hi rows and lo rows `half` rows further
// (split_scaled); the tensor-core projection multiplies its results by
// 1/rms itself.  grid (ceil(H / 2048), B), 256 threads x 8 elements.
__global__ void __launch_bounds__(256) scale_split_kernel(const void *x, int x_f32, const float *gamma, int H,
                                                          __nv_bfloat16 *xs, int half) {
    TPL_TRACE_VARS
    if (threadIdx.x == 0) TPL_TRACE_AT(0);
    pdl_wait();
    pdl_trigger();
    if (threadIdx.x == 0) {
        TPL_TRACE_AT(1);
        TPL_TRACE_AT(2);
        TPL_TRACE_AT(3);
        TPL_TRACE_PUT(TR_OPERAND);
    }
    const int64_t row = blockIdx.y;
    const int c = blockIdx.x * 256 + threadIdx.x;
    if (8 * c >= H) return;
    float v[8];
    if (x_f32) {
        const float4 *p = reinterpret_cast<const float4 *>(static_cast<const float *>(x) + row * H + 8 * c);
        const float4 u0 = p[0], u1 = p[1];
        v[0] = u0.x; v[1] = u0.y; v[2] = u0.z; v[3] = u0.w; v[4] = u1.x; v[5] = u1.y; v[6] = u1.z; v[7] = u1.w;
    } else {
        const uint4 u = *reinterpret_cast<const uint4 *>(static_cast<const __nv_bfloat16 *>(x) + row * H + 8 * c);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            v[2 * e] = bf16lo(w[e]);
            v[2 * e + 1] = bf16hi(w[e]);
        }
    }
    __align__(16) __nv_bfloat16 h8[8], l8[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) split_scaled(v[e], gamma, 8 * c + e, h8[e], l8[e]);
    *reinterpret_cast<uint4 *>(xs + row * H + 8 * c) = *reinterpret_cast<const uint4 *>(h8);
    *reinterpret_cast<uint4 *>(xs + (row + half) * H + 8 * c) = *reinterpret_cast<const uint4 *>(l8);
}

}  // namespace tpl
