// Device helpers shared by the kernels (one translation unit includes them).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace tpl {

// Error word of this library on the current device (recorded by kernels that
// detect an inconsistency; read and cleared by tpl_last_device_error).
__device__ unsigned int g_err_word;

__device__ __forceinline__ void record_error(unsigned code) { atomicOr(&g_err_word, code); }

// Programmatic dependent launch: wait for the preceding grid's results /
// allow the next grid to be scheduled.  Both are no-ops when the launch did
// not opt in.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Timeline tracing (built only with -DTPL_TRACE, the library's diagnostic
// variant): one thread per CTA takes up to four global-timer marks (entry,
// dependency wait passed, main loop done, exit) and appends one record per
// CTA; tpl_trace_read copies the records out.  Compiled out otherwise.
enum { TR_QKV = 1, TR_ATTN = 2, TR_O = 3, TR_GU = 4, TR_DOWN = 5, TR_OPERAND = 6, TR_REDUCE = 7 };
#ifdef TPL_TRACE
constexpr unsigned kTraceMax = 1u << 18;
struct TraceRec {
    uint32_t tag, cta, smid, grid;
    uint64_t t[4];
};
__device__ TraceRec g_trace[kTraceMax];
__device__ unsigned g_trace_n;
__device__ __forceinline__ uint64_t trace_now() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
__device__ __forceinline__ void trace_put(uint32_t tag, const uint64_t (&t)[4]) {
    uint32_t sm;
    asm volatile("mov.u32 %0, %%smid;" : "=r"(sm));
    const unsigned k = atomicAdd(&g_trace_n, 1u);
    if (k < kTraceMax) {
        TraceRec r;
        r.tag = tag;
        r.cta = blockIdx.x + gridDim.x * blockIdx.y;
        r.smid = sm;
        r.grid = gridDim.x * gridDim.y;
        r.t[0] = t[0];
        r.t[1] = t[1];
        r.t[2] = t[2];
        r.t[3] = t[3];
        g_trace[k] = r;
    }
}
#define TPL_TRACE_VARS uint64_t tr_t[4] = {0, 0, 0, 0};
#define TPL_TRACE_AT(i) (tr_t[i] = trace_now())
#define TPL_TRACE_PUT(tag) trace_put((tag), tr_t)
#else
#define TPL_TRACE_VARS
#define TPL_TRACE_AT(i) ((void)0)
#define TPL_TRACE_PUT(tag) ((void)0)
#endif

// 16-byte streaming load of read-once data (weights, KV cache): not kept in L1,
// first out of L2 under the given policy.
__device__ __forceinline__ uint4 ldg_stream(const void *p, uint64_t policy) {
    uint4 r;
    asm("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0,%1,%2,%3}, [%4], %5;"
        : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
        : "l"(p), "l"(policy));
    return r;
}

// L2 policy for data read exactly once (weights and KV-cache streams): evict
// it first, so that it does not push out the small data read again
// (activations, cross-CTA partials, norms).
__device__ __forceinline__ uint64_t evict_first_policy() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

__device__ __forceinline__ void prefetch_l2(const void *p) { asm volatile("prefetch.global.L2 [%0];" ::"l"(p)); }

__device__ __forceinline__ uint4 lds128(const void *p) {
    uint4 r;
    unsigned a = (unsigned)__cvta_generic_to_shared(p);
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "r"(a));
    return r;
}

// D += A(16x16, row) * B(16x8, col), bf16 inputs, fp32 accumulate.
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ float bf16lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }

// Round-to-nearest-even packing of two floats into bf16x2 (lo in low half).
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
    return r;
}

__device__ __forceinline__ float load_act(const void *p, int is_f32, int64_t i) {
    return is_f32 ? static_cast<const float *>(p)[i]
                  : __bfloat162float(static_cast<const __nv_bfloat16 *>(p)[i]);
}

__device__ __forceinline__ void store_act(void *p, int is_f32, int64_t i, float v) {
    if (is_f32) static_cast<float *>(p)[i] = v;
    else static_cast<__nv_bfloat16 *>(p)[i] = __float2bfloat16_rn(v);
}

__device__ __forceinline__ float silu(float z) { return z / (1.0f + expf(-z)); }

// The operand of the tensor-core decode projections: a = v * gamma[i] (v
// without gamma), as bf16 hi = rn(a) and lo = rn(a - hi).  Written with
// explicit roundings so that every kernel producing it gives the same bits.
__device__ __forceinline__ void split_scaled(float v, const float *gamma, int64_t i, __nv_bfloat16 &hi,
                                             __nv_bfloat16 &lo) {
    const float a = gamma ? __fmul_rn(v, gamma[i]) : v;
    hi = __float2bfloat16_rn(a);
    lo = __float2bfloat16_rn(__fsub_rn(a, __bfloat162float(hi)));
}

// cos and sin of the rotary angle pos * theta.  The angle is formed and
// brought into [-pi, pi] in fp64 (positions of long sequences give angles of
// thousands of radians, where fp32 would lose the low bits), then evaluated
// by the hardware's fp32 approximation, whose absolute error on [-pi, pi]
// (a few 1e-7) is far below the bf16 rounding the rotated values meet.
__device__ __forceinline__ void rope_cs(double pos, double theta, float &c, float &s) {
    const double ang = pos * theta;
    const double r = ang - 6.283185307179586 * rint(ang * 0.15915494309189535);
    __sincosf((float)r, &s, &c);
}

// Asynchronous 16-byte global -> shared copies and ldmatrix fragment loads.
__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((unsigned)__cvta_generic_to_shared(dst)), "l"(src)
                 : "memory");
}
// The same with an L2 cache policy (createpolicy), for streams read once.
__device__ __forceinline__ void cp_async16_hint(void *dst, const void *src, uint64_t policy) {
    asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2;" ::"r"(
                     (unsigned)__cvta_generic_to_shared(dst)),
                 "l"(src), "l"(policy)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_1() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_0() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ void ldsm_x4(const void *p, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"((unsigned)__cvta_generic_to_shared(p)));
}
__device__ __forceinline__ void ldsm_x4_t(const void *p, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"((unsigned)__cvta_generic_to_shared(p)));
}


}  // namespace tpl
