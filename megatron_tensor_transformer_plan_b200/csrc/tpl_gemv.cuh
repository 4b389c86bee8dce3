// Matrix-vector kernels for the decode projections (B <= 16 tokens).
//
// One CTA per SM (512 threads).  The grid is rb row blocks x ksplit K-splits.
// Inside a CTA the 16 warps form wk K-groups x wr row slots; a warp streams
// 8-row groups of the weight matrix over its K-group's 128-column blocks with
// 16-byte loads, double-buffered in registers, against the activation slice
// the CTA staged (normalised, rounded to the activation type) in shared
// memory.  Partial sums per (K-group, row, token) land in shared memory and
// are added in a fixed order per segment (shard) at the end of each round of
// row groups; split-K CTAs hand their per-segment partials to the last CTA of
// the row block to arrive (an arrival counter, no waiting), which adds them
// in order.  The per-segment sums p_s are the shard partials of the row-split
// projections ("Tensor parallel scaling curves", "What tensor parallelism
// actually splits"): the fused epilogue adds them in ascending shard order,
// the separate mode writes them out for tpl_reduce_partials, which adds them
// in the same order -- so both modes give identical bits.
//
// Inner product modes:
// Weight rows are padded to whole 128-column blocks in the packed layout, and
// each warp keeps two blocks of loads in flight in a register ring (deeper
// rings measured slower: register pressure).
//
//   MODE 0 -- bf16 weights on the tensor cores (mma.sync m16n8k16): the
//             activation tile is the A operand (tokens as rows), 8 weight rows
//             the B operand; the k index of each 16-wide step is permuted so
//             that every lane's operands are 16-byte contiguous in memory.
//   MODE 1 -- fp32 weights with fp32 FFMA (exact-arithmetic comparison mode).
//   MODE 2 -- bf16 weights with FFMA on the CUDA cores (kept to measure
//             against MODE 0).
//   MODE 3 -- MODE 0 with each activation value carried as two bf16 parts
//             (hi = bf16(v), lo = bf16(v - hi)), staged as token rows B..2B-1;
//             for B <= 8 the lo parts ride in the otherwise-zero A rows 8-15
//             of the same mma, for B > 8 they take a second mma.  Used where
//             the result feeds a softmax (the Q projection).
#pragma once

#include "tpl_common.cuh"
#include "tpl_internal.h"

namespace tpl {

enum { EPI_QKV = 0, EPI_GU = 1, EPI_ROW = 2, EPI_ROW_PARTIAL = 3 };

// How far (blocks per warp) an L2 prefetch runs ahead of the register loads:
// issued before the dependency wait for the first blocks, then one block per
// block loaded.  The register ring holds 2 blocks per warp (64 KB per SM in
// flight), too few to cover DRAM latency alone; on the 7B layer at one token
// distances of 2-3 took 99.9-100.6 us, 4 took 102.8, 8 took 108.9, 16 took
// 115.1, and no in-loop prefetch 112.9.
constexpr int kPrefetchBlocks = 3;

struct GemvArgs {
    const char *W;   // first weight block
    int64_t blk_r;   // bytes between row blocks (column-parallel shards)
    int64_t blk_s;   // bytes between K segments (row-parallel shards)
    int rps;         // rows per row block
    int ldw;         // elements per weight row inside a block
    GemvGeom g;
    int B;
    const void *x;   // activation source [B][ldx]; column seg*Kseg + k
    int x_f32, ldx;
    int norm;
    const float *gamma;
    float eps;
    int epi;
    float *out32;
    void *out_act;
    int act_f32;
    const void *resid;
    int resid_f32;
    float *partials;  // [nseg][B][N]
    float *q;
    float *knew, *vnew;  // [B][n_kv][hd] fp32 copies of the new k/v, or NULL
    __nv_bfloat16 *kc, *vc;
    int nq, nq_s, nkv_s, hd, batch_cap;
    int64_t S, seq_cap;
    float *gp;
    unsigned *tickets;
    int trace_row_tag;  // timeline tag of a row-parallel launch (traced builds)
};

template <int MODE>
struct GemvTraits;
// WES / XES: weight / staged-activation element bytes; LPM: 16-byte loads per
// lane per 32-column step.
template <>
struct GemvTraits<0> {  // bf16 weights, bf16 staged x, tensor cores
    static constexpr int WES = 2, XES = 2, LPM = 1;
};
template <>
struct GemvTraits<1> {  // fp32 weights, fp32 staged x, FFMA
    static constexpr int WES = 4, XES = 4, LPM = 2;
};
template <>
struct GemvTraits<2> {  // bf16 weights, bf16 staged x, FFMA
    static constexpr int WES = 2, XES = 2, LPM = 1;
};
template <>
struct GemvTraits<3> {  // MODE 0 with the activation carried as bf16 hi + lo
    static constexpr int WES = 2, XES = 2, LPM = 1;
};

// Segment sums and the final write for one (row, token).
struct SegSums {
    float p[8];
};

__device__ __forceinline__ void gemv_final_row(const GemvArgs &a, int row, int tok, const SegSums &ss) {
    const int N = a.g.N, B = a.B;
    if (a.epi == EPI_QKV) {
        const float v = ss.p[0];
        const int s = row / a.rps, l = row % a.rps;
        const int qd = a.nq_s * a.hd, kd = a.nkv_s * a.hd;
        if (l < qd) {
            const int head = s * a.nq_s + l / a.hd, dim = l % a.hd;
            a.q[((int64_t)tok * a.nq + head) * a.hd + dim] = v;
        } else {
            const bool isk = l < qd + kd;
            const int ll = isk ? l - qd : l - qd - kd;
            const int kvl = ll / a.hd, dim = ll % a.hd;
            __nv_bfloat16 *c = isk ? a.kc : a.vc;
            c[((((int64_t)s * a.batch_cap + tok) * a.nkv_s + kvl) * a.seq_cap + a.S) * a.hd + dim] =
                __float2bfloat16_rn(v);
            float *f = isk ? a.knew : a.vnew;
            if (f) f[((int64_t)tok * (a.nkv_s * (a.nq / a.nq_s)) + s * a.nkv_s + kvl) * a.hd + dim] = v;
        }
    } else if (a.epi == EPI_ROW) {
        float acc = ss.p[0];
        for (int s = 1; s < a.g.nseg; ++s) acc = acc + ss.p[s];
        if (a.resid) acc = load_act(a.resid, a.resid_f32, (int64_t)tok * N + row) + acc;
        if (a.out32) a.out32[(int64_t)tok * N + row] = acc;
        if (a.out_act) store_act(a.out_act, a.act_f32, (int64_t)tok * N + row, acc);
    } else {  // EPI_ROW_PARTIAL
        for (int s = 0; s < a.g.nseg; ++s) a.partials[((int64_t)s * B + tok) * N + row] = ss.p[s];
    }
}

__device__ __forceinline__ void gemv_final_pair(const GemvArgs &a, int pair, int tok, float gsum, float usum) {
    store_act(a.out_act, a.act_f32, (int64_t)tok * (a.g.N / 2) + pair, silu(gsum) * usum);
}

template <int MODE, bool BIG>  // BIG: more than 8 tokens (tokens 8..15 in A rows 8-15)
__global__ void __launch_bounds__(kGemvThreads, 1) gemv_kernel(const __grid_constant__ GemvArgs a) {
    using T = GemvTraits<MODE>;
    constexpr bool XSPLIT = MODE == 3;
    constexpr bool MMA = MODE == 0 || MODE == 3;
    constexpr int D = 2;                       // blocks in flight per warp (register ring)
    constexpr int NW = 4 * T::LPM;             // uint4 per block per lane
    constexpr int BLK_BYTES = 128 * T::WES;    // one 128-column block of one row
    extern __shared__ __align__(128) unsigned char smem[];
    const GemvGeom &g = a.g;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int gid = lane >> 2, c = lane & 3;
    const int B = a.B;
    const int rb = blockIdx.x / g.ksplit, ks = blockIdx.x % g.ksplit;
    const int rg0 = (int)((int64_t)rb * g.ng / g.rb), rg1 = (int)((int64_t)(rb + 1) * g.ng / g.rb);
    const int kgl = warp % g.wk, wslot = warp / g.wk;
    TPL_TRACE_VARS
    if (tid == 0) TPL_TRACE_AT(0);

    // K-group -> segment and block range.
    const int KG = g.ksplit * g.wk;
    const int kpseg = KG / g.nseg;
    const int Gk = ks * g.wk + kgl;
    const int seg = Gk / kpseg, piece = Gk % kpseg;
    const int kb_lo = (int)((int64_t)piece * g.nb / kpseg), kb_hi = (int)((int64_t)(piece + 1) * g.nb / kpseg);
    // CTA's staged span.
    const int seg_lo = (ks * g.wk) / kpseg;
    int cblk_lo = 0, nbc = g.nb;
    if (g.ksplit > g.nseg) {
        const int per = g.pieces, pi = ks % per;
        cblk_lo = (int)((int64_t)pi * g.nb / per);
        nbc = (int)((int64_t)(pi + 1) * g.nb / per) - cblk_lo;
    }
    const int kpc = g.wk / g.segs_per_cta;  // K-groups per segment inside the CTA

    unsigned char *xs = smem;
    const size_t lo_off = (size_t)B * g.x_stride;  // hi+lo staging: lo rows follow the hi rows
    float *part = reinterpret_cast<float *>(smem + (size_t)(XSPLIT ? 2 : 1) * B * g.x_stride);
    const int prows = g.wr * g.rgc * 8;  // rows per round
    float *s_inv = part + (size_t)g.wk * prows * B;
    int *s_flag = reinterpret_cast<int *>(s_inv + 16);

    // Warp's work: row groups r = 0..nrg_w-1 (rg = rg0 + wslot + r*wr), each
    // nblk blocks of its K-group; T blocks in all, streamed in that order.
    const int nrg_w = rg1 - rg0 > wslot ? (rg1 - rg0 - wslot + g.wr - 1) / g.wr : 0;
    const int nblk = kb_hi - kb_lo;
    const int T_blocks = nrg_w * nblk;
    // weights are padded to whole 128-column blocks and N is a multiple of 8:
    // every load below is in range without a predicate.
    auto rowptr = [&](int r) -> const char * {
        const int row = (rg0 + wslot + r * g.wr) * 8 + gid;
        return a.W + (int64_t)(row / a.rps) * a.blk_r + (int64_t)seg * a.blk_s +
               ((int64_t)(row % a.rps) * a.ldw + (int64_t)kb_lo * 128 + 8 * c) * T::WES;
    };
    uint4 ring[D][NW];
    const uint64_t wpol = evict_first_policy();  // the weights are read once
    int lr = 0, lj = 0;
    const char *lptr = nrg_w > 0 ? rowptr(0) : a.W;
    auto load_next = [&](uint4 (&w)[NW]) {
#pragma unroll
        for (int m = 0; m < 4; ++m)
#pragma unroll
            for (int l = 0; l < T::LPM; ++l) w[m * T::LPM + l] = ldg_stream(lptr + m * 32 * T::WES + 16 * l, wpol);
        if (++lj == nblk) {
            lj = 0;
            if (++lr < nrg_w) lptr = rowptr(lr);
        } else {
            lptr += BLK_BYTES;
        }
    };
    // Issue the first weight loads before waiting on the previous kernel, and
    // prefetch the next kPrefetchBlocks blocks of this warp's stream into L2
    // (each block: 8 rows x 128 columns; lanes with c == 0 cover both 128-byte
    // lines of their row); the loop keeps that distance.
#pragma unroll
    for (int d = 0; d < D; ++d)
        if (d < T_blocks) load_next(ring[d]);
    // L2 prefetch cursor (row group pr, block pj)
    int pr = lr, pj = lj;
    const char *pp = lptr;
    auto prefetch_next = [&]() {
        if (pr >= nrg_w) return;
        if (c == 0) {
            prefetch_l2(pp);
            prefetch_l2(pp + 64 * T::WES);
            if (T::WES == 4) {
                prefetch_l2(pp + 128 * 2);
                prefetch_l2(pp + 128 * 3);
            }
        }
        if (++pj == nblk) {
            pj = 0;
            if (++pr < nrg_w) pp = rowptr(pr);
        } else {
            pp += BLK_BYTES;
        }
    };
    for (int q = 0; q < kPrefetchBlocks && D + q < T_blocks; ++q) prefetch_next();
    pdl_wait();
    pdl_trigger();
    if (tid == 0) TPL_TRACE_AT(1);

    // ---- stage the activation slice (normalised if requested) ----
    // Each token gets a power-of-two group of tpt threads (512 / next pow2 of
    // B), so chunk coordinates are shifts and masks.  A chunk is 8 elements.
    auto load8 = [&](int64_t src, float (&v)[8]) {
        if (a.x_f32) {
            const float4 *p4 = reinterpret_cast<const float4 *>(static_cast<const float *>(a.x) + src);
            const float4 x0 = p4[0], x1 = p4[1];
            v[0] = x0.x; v[1] = x0.y; v[2] = x0.z; v[3] = x0.w;
            v[4] = x1.x; v[5] = x1.y; v[6] = x1.z; v[7] = x1.w;
        } else {
            const uint4 r4 = *reinterpret_cast<const uint4 *>(static_cast<const __nv_bfloat16 *>(a.x) + src);
            v[0] = bf16lo(r4.x); v[1] = bf16hi(r4.x); v[2] = bf16lo(r4.y); v[3] = bf16hi(r4.y);
            v[4] = bf16lo(r4.z); v[5] = bf16hi(r4.z); v[6] = bf16lo(r4.w); v[7] = bf16hi(r4.w);
        }
    };
    // store one normalised chunk (tok, smem column col) as bf16 (+ lo part) or fp32
    auto store8 = [&](int tok, int col, const float (&v)[8]) {
        unsigned char *dst = xs + (size_t)tok * g.x_stride + (size_t)col * T::XES;
        if (T::XES == 2) {
            uint4 o;
            o.x = pack_bf16x2(v[0], v[1]); o.y = pack_bf16x2(v[2], v[3]);
            o.z = pack_bf16x2(v[4], v[5]); o.w = pack_bf16x2(v[6], v[7]);
            *reinterpret_cast<uint4 *>(dst) = o;
            if constexpr (XSPLIT) {
                uint4 l;
                l.x = pack_bf16x2(v[0] - bf16lo(o.x), v[1] - bf16hi(o.x));
                l.y = pack_bf16x2(v[2] - bf16lo(o.y), v[3] - bf16hi(o.y));
                l.z = pack_bf16x2(v[4] - bf16lo(o.z), v[5] - bf16hi(o.z));
                l.w = pack_bf16x2(v[6] - bf16lo(o.w), v[7] - bf16hi(o.w));
                *reinterpret_cast<uint4 *>(dst + lo_off) = l;
            }
        } else {
            reinterpret_cast<float4 *>(dst)[0] = make_float4(v[0], v[1], v[2], v[3]);
            reinterpret_cast<float4 *>(dst)[1] = make_float4(v[4], v[5], v[6], v[7]);
        }
    };
    auto scale8 = [&](int k, float inv, float (&v)[8]) {
        const float4 g0 = __ldg(reinterpret_cast<const float4 *>(a.gamma + k));
        const float4 g1 = __ldg(reinterpret_cast<const float4 *>(a.gamma + k) + 1);
        v[0] *= inv * g0.x; v[1] *= inv * g0.y; v[2] *= inv * g0.z; v[3] *= inv * g0.w;
        v[4] *= inv * g1.x; v[5] *= inv * g1.y; v[6] *= inv * g1.z; v[7] *= inv * g1.w;
    };
    const int lgBp = B <= 1 ? 0 : 32 - __clz(B - 1);  // log2 of the next power of two >= B
    const int lg_tpt = 9 - lgBp;                       // kGemvThreads = 512 = 2^9
    const int tpt = 1 << lg_tpt, tok_me = tid >> lg_tpt, lt = tid & (tpt - 1);
    const bool tok_ok = tok_me < B;
    const int64_t xrow = (int64_t)tok_me * a.ldx;
    const int chunks_seg = nbc * 16;                   // staged chunks per segment
    float *s_red = part;                               // scratch: per-warp sums of squares
    const int wpt = tpt >> 5;                          // warps per token
    // full-row, one-pass case: column-parallel, whole row staged, the raw
    // loads held in 32 registers (8 bf16 chunks or 4 fp32 chunks per thread)
    const int cpt_full = a.ldx >> 3;
    const int hold = a.x_f32 ? 4 : 8;
    const bool one_pass = a.norm && g.nseg == 1 && g.ksplit == 1 && cpt_full <= hold * tpt;
    if (one_pass) {
        uint4 raw[8];  // bf16: 8 chunks; fp32: 4 chunks as pairs (raw[2q], raw[2q+1])
#pragma unroll
        for (int q = 0; q < 8; ++q) raw[q] = make_uint4(0, 0, 0, 0);
        if (a.x_f32) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int c16 = lt + q * tpt;
                if (tok_ok && c16 < cpt_full) {
                    const uint4 *p4 = reinterpret_cast<const uint4 *>(static_cast<const float *>(a.x) + xrow + (int64_t)c16 * 8);
                    raw[2 * q] = p4[0];
                    raw[2 * q + 1] = p4[1];
                }
            }
        } else {
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const int c16 = lt + q * tpt;
                if (tok_ok && c16 < cpt_full)
                    raw[q] = *reinterpret_cast<const uint4 *>(static_cast<const __nv_bfloat16 *>(a.x) + xrow + (int64_t)c16 * 8);
            }
        }
        auto unpack = [&](int q, float (&v)[8]) {
            if (a.x_f32) {
                const uint4 r0 = raw[2 * q], r1 = raw[2 * q + 1];
                v[0] = __uint_as_float(r0.x); v[1] = __uint_as_float(r0.y); v[2] = __uint_as_float(r0.z); v[3] = __uint_as_float(r0.w);
                v[4] = __uint_as_float(r1.x); v[5] = __uint_as_float(r1.y); v[6] = __uint_as_float(r1.z); v[7] = __uint_as_float(r1.w);
            } else {
                const uint4 r4 = raw[q];
                v[0] = bf16lo(r4.x); v[1] = bf16hi(r4.x); v[2] = bf16lo(r4.y); v[3] = bf16hi(r4.y);
                v[4] = bf16lo(r4.z); v[5] = bf16hi(r4.z); v[6] = bf16lo(r4.w); v[7] = bf16hi(r4.w);
            }
        };
        float ss = 0.f;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            if (q < hold) {
                float v[8];
                unpack(q, v);
#pragma unroll
                for (int e = 0; e < 8; ++e) ss += v[e] * v[e];
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        if (lane == 0) s_red[warp] = ss;
        __syncthreads();
        float tot = 0.f;
        for (int w = 0; w < wpt; ++w) tot += s_red[tok_me * wpt + w];  // fixed order
        const float inv = 1.0f / sqrtf(tot / (float)a.ldx + a.eps);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const int c16 = lt + q * tpt;
            if (q < hold && tok_ok && c16 < nbc * 16) {
                float v[8];
                unpack(q, v);  // zeros past the row end
                if (c16 < cpt_full) scale8(c16 * 8, inv, v);
                store8(tok_me, c16 * 8, v);
            }
        }
        // padding chunks not covered above (only when the row is padded)
        for (int c16 = lt + hold * tpt; tok_ok && c16 < nbc * 16; c16 += tpt) {
            float z[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            store8(tok_me, c16 * 8, z);
        }
    } else {
        float inv = 1.f;
        if (a.norm) {
            float ss = 0.f;
            for (int c0 = lt; c0 < cpt_full; c0 += 4 * tpt) {
                float v[4][8];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int c16 = c0 + q * tpt;
                    if (tok_ok && c16 < cpt_full) load8(xrow + (int64_t)c16 * 8, v[q]);
                    else {
#pragma unroll
                        for (int e = 0; e < 8; ++e) v[q][e] = 0.f;
                    }
                }
#pragma unroll
                for (int q = 0; q < 4; ++q)
#pragma unroll
                    for (int e = 0; e < 8; ++e) ss += v[q][e] * v[q][e];
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
            if (lane == 0) s_red[warp] = ss;
            __syncthreads();
            float tot = 0.f;
            for (int w = 0; w < wpt; ++w) tot += s_red[tok_me * wpt + w];
            inv = 1.0f / sqrtf(tot / (float)a.ldx + a.eps);
        }
        if (tok_ok) {
            for (int sl = 0; sl < g.segs_per_cta; ++sl) {
                const int64_t srow = xrow + (int64_t)(seg_lo + sl) * g.Kseg + (int64_t)cblk_lo * 128;
                const int kbase = cblk_lo * 128;
                for (int c0 = lt; c0 < chunks_seg; c0 += 4 * tpt) {
                    float v[4][8];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int c16 = c0 + q * tpt;
                        if (c16 < chunks_seg && kbase + c16 * 8 < g.Kseg) load8(srow + (int64_t)c16 * 8, v[q]);
                        else {
#pragma unroll
                            for (int e = 0; e < 8; ++e) v[q][e] = 0.f;
                        }
                    }
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int c16 = c0 + q * tpt;
                        if (c16 < chunks_seg) {
                            if (a.norm && kbase + c16 * 8 < g.Kseg) scale8(kbase + c16 * 8, inv, v[q]);
                            store8(tok_me, sl * chunks_seg * 8 + c16 * 8, v[q]);
                        }
                    }
                }
            }
        }
    }
    __syncthreads();

    // ---- main loop ----
    const int rg_cta = rg1 - rg0;
    const int rounds = (((rg_cta + g.wr - 1) / g.wr) + g.rgc - 1) / g.rgc;
    const int sl_mine = seg - seg_lo;  // this warp's segment inside the CTA
    // this lane's activation bytes for block j of the K-group: xlane + j * 128 * XES
    const unsigned char *xlane =
        xs + (size_t)gid * g.x_stride + ((size_t)(sl_mine * nbc + kb_lo - cblk_lo) * 128 + 8 * c) * T::XES;
    float acc[MMA ? 4 : 16];
#pragma unroll
    for (int i = 0; i < (MMA ? 4 : 16); ++i) acc[i] = 0.f;

    // one block (8 rows x 128 columns) against the staged activations
    auto compute = [&](const uint4 (&w)[NW], int j) {
        const unsigned char *xp = xlane + (size_t)j * 128 * T::XES;
        if constexpr (MODE == 0) {
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const uint4 xa = (BIG || gid < B) ? lds128(xp + 64 * m) : make_uint4(0, 0, 0, 0);
                const uint4 xb = (BIG && gid + 8 < B) ? lds128(xp + 8 * g.x_stride + 64 * m) : make_uint4(0, 0, 0, 0);
                mma_bf16_16816(acc, xa.x, xb.x, xa.y, xb.y, w[m].x, w[m].y);
                mma_bf16_16816(acc, xa.z, xb.z, xa.w, xb.w, w[m].z, w[m].w);
            }
        } else if constexpr (MODE == 3) {
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                if constexpr (!BIG) {
                    // rows gid: hi of token gid, rows gid+8: lo of token gid
                    uint4 xa = make_uint4(0, 0, 0, 0), xb = make_uint4(0, 0, 0, 0);
                    if (gid < B) {
                        xa = lds128(xp + 64 * m);
                        xb = lds128(xp + lo_off + 64 * m);
                    }
                    mma_bf16_16816(acc, xa.x, xb.x, xa.y, xb.y, w[m].x, w[m].y);
                    mma_bf16_16816(acc, xa.z, xb.z, xa.w, xb.w, w[m].z, w[m].w);
                } else {
#pragma unroll
                    for (int part_i = 0; part_i < 2; ++part_i) {
                        const unsigned char *pp = xp + (part_i ? lo_off : 0) + 64 * m;
                        const uint4 xa = lds128(pp);
                        const uint4 xb = gid + 8 < B ? lds128(pp + 8 * g.x_stride) : make_uint4(0, 0, 0, 0);
                        mma_bf16_16816(acc, xa.x, xb.x, xa.y, xb.y, w[m].x, w[m].y);
                        mma_bf16_16816(acc, xa.z, xb.z, xa.w, xb.w, w[m].z, w[m].w);
                    }
                }
            }
        } else {
            // FFMA: lane (gid, c) owns row gid, columns 32m + 8c .. +8
            const unsigned char *xt = xp - (size_t)gid * g.x_stride;  // token rows start here
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                float wv[8];
                if constexpr (T::WES == 4) {
                    const uint4 w0 = w[m * 2], w1 = w[m * 2 + 1];
                    wv[0] = __uint_as_float(w0.x); wv[1] = __uint_as_float(w0.y);
                    wv[2] = __uint_as_float(w0.z); wv[3] = __uint_as_float(w0.w);
                    wv[4] = __uint_as_float(w1.x); wv[5] = __uint_as_float(w1.y);
                    wv[6] = __uint_as_float(w1.z); wv[7] = __uint_as_float(w1.w);
                } else {
                    const uint4 w0 = w[m];
                    wv[0] = bf16lo(w0.x); wv[1] = bf16hi(w0.x); wv[2] = bf16lo(w0.y); wv[3] = bf16hi(w0.y);
                    wv[4] = bf16lo(w0.z); wv[5] = bf16hi(w0.z); wv[6] = bf16lo(w0.w); wv[7] = bf16hi(w0.w);
                }
#pragma unroll
                for (int tok = 0; tok < 16; ++tok) {
                    if (tok < B) {
                        float xv[8];
                        const unsigned char *xq = xt + (size_t)tok * g.x_stride + 32 * m * T::XES;
                        if constexpr (T::XES == 4) {
                            const uint4 x0 = lds128(xq), x1 = lds128(xq + 16);
                            xv[0] = __uint_as_float(x0.x); xv[1] = __uint_as_float(x0.y);
                            xv[2] = __uint_as_float(x0.z); xv[3] = __uint_as_float(x0.w);
                            xv[4] = __uint_as_float(x1.x); xv[5] = __uint_as_float(x1.y);
                            xv[6] = __uint_as_float(x1.z); xv[7] = __uint_as_float(x1.w);
                        } else {
                            const uint4 x0 = lds128(xq);
                            xv[0] = bf16lo(x0.x); xv[1] = bf16hi(x0.x); xv[2] = bf16lo(x0.y); xv[3] = bf16hi(x0.y);
                            xv[4] = bf16lo(x0.z); xv[5] = bf16hi(x0.z); xv[6] = bf16lo(x0.w); xv[7] = bf16hi(x0.w);
                        }
                        float sacc = acc[tok];
#pragma unroll
                        for (int e = 0; e < 8; ++e) sacc = fmaf(wv[e], xv[e], sacc);
                        acc[tok] = sacc;
                    }
                }
            }
        }
    };

    // partial sums of one finished row group for this K-group
    auto write_part = [&](int r, int k) {
        const int pr = (wslot + (k - r * g.rgc) * g.wr) * 8;
        float *pp = part + ((size_t)kgl * prows + pr) * B;
        if constexpr (MMA) {
            if (XSPLIT && !BIG) {
                // hi and lo halves of the same token
                acc[0] += acc[2];
                acc[1] += acc[3];
                acc[2] = acc[3] = 0.f;
            }
            if (gid < B) {
                pp[(2 * c) * B + gid] = acc[0];
                pp[(2 * c + 1) * B + gid] = acc[1];
            }
            if (BIG && gid + 8 < B) {
                pp[(2 * c) * B + gid + 8] = acc[2];
                pp[(2 * c + 1) * B + gid + 8] = acc[3];
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[i] = 0.f;
        } else {
#pragma unroll
            for (int tok = 0; tok < 16; ++tok) {
                float sacc = acc[tok];
                sacc += __shfl_xor_sync(0xffffffffu, sacc, 1);
                sacc += __shfl_xor_sync(0xffffffffu, sacc, 2);
                if (tok < B && (tok & 3) == c) pp[gid * B + tok] = sacc;
                acc[tok] = 0.f;
            }
        }
    };

    int i = 0;          // next block to consume
    int cr = 0, cj = 0; // its row group and block within the K-group
    for (int r = 0; r < rounds; ++r) {
        const int k_end = min((r + 1) * g.rgc, nrg_w);
        if (nblk == 0) {
            // an empty K-group contributes zeros
            for (int k = r * g.rgc; k < k_end; ++k) write_part(r, k);
        }
        const int i_end = k_end * nblk;
        // rounds hold a multiple of D blocks (rgc is a multiple of 4), so the
        // ring slot of block i is always i % D
        for (; i < i_end; i += D) {
#pragma unroll
            for (int d = 0; d < D; ++d) {
                if (i + d < i_end) {
                    compute(ring[d], cj);
                    if (i + d + D < T_blocks) {
                        load_next(ring[d]);
                        prefetch_next();
                    }
                    if (++cj == nblk) {
                        write_part(r, cr);
                        cj = 0;
                        ++cr;
                    }
                }
            }
        }
        __syncthreads();
        // ---- round epilogue: fixed-order sums over K-groups per segment ----
        const int rbase = (rg0 + r * g.wr * g.rgc) * 8;
        const int nrows = min(prows, min(rg1 * 8, g.N) - rbase);
        if (nrows > 0) {
            const int pr_ok = g.ksplit == 1;
            const int pc = g.ksplit > g.nseg ? ks % g.pieces : 0;
            if (a.epi == EPI_GU) {
                for (int u = tid; u < (nrows / 2) * B; u += kGemvThreads) {
                    const int pp = u / B, tok = u % B;
                    float gs = 0.f, us = 0.f;
                    for (int kg = 0; kg < g.wk; ++kg) {
                        gs += part[((size_t)kg * prows + 2 * pp) * B + tok];
                        us += part[((size_t)kg * prows + 2 * pp + 1) * B + tok];
                    }
                    const int row = rbase + 2 * pp;
                    if (pr_ok) {
                        gemv_final_pair(a, row / 2, tok, gs, us);
                    } else {
                        a.gp[(((int64_t)0 * g.pieces + pc) * g.N + row) * B + tok] = gs;
                        a.gp[(((int64_t)0 * g.pieces + pc) * g.N + row + 1) * B + tok] = us;
                    }
                }
            } else {
                for (int u = tid; u < nrows * B; u += kGemvThreads) {
                    const int prow = u / B, tok = u % B;
                    const int row = rbase + prow;
                    SegSums ss;
                    for (int sl = 0; sl < g.segs_per_cta; ++sl) {
                        float sv = 0.f;
                        for (int kg = sl * kpc; kg < (sl + 1) * kpc; ++kg) sv += part[((size_t)kg * prows + prow) * B + tok];
                        ss.p[sl] = sv;
                    }
                    if (pr_ok) {
                        gemv_final_row(a, row, tok, ss);
                    } else {
                        for (int sl = 0; sl < g.segs_per_cta; ++sl)
                            a.gp[(((int64_t)(seg_lo + sl) * g.pieces + pc) * g.N + row) * B + tok] = ss.p[sl];
                    }
                }
            }
        }
        __syncthreads();
    }

    // ---- split-K: the last CTA of the row block adds the partials in order ----
    if (tid == 0) TPL_TRACE_AT(2);
    if (g.ksplit > 1) {
        __threadfence();
        __syncthreads();
        if (tid == 0) {
            const unsigned prev = atomicAdd(&a.tickets[rb], 1u);
            *s_flag = prev == (unsigned)(g.ksplit - 1);
            if (prev >= (unsigned)g.ksplit) record_error(1u);
        }
        __syncthreads();
        if (*s_flag) {
            __threadfence();
            const int row0 = rg0 * 8, row1 = min(rg1 * 8, g.N);
            if (a.epi == EPI_GU) {
                for (int u = tid; u < ((row1 - row0) / 2) * B; u += kGemvThreads) {
                    const int row = row0 + 2 * (u / B), tok = u % B;
                    float gs = 0.f, us = 0.f;
                    for (int pc = 0; pc < g.pieces; ++pc) {
                        gs += __ldcg(&a.gp[(((int64_t)pc) * g.N + row) * B + tok]);
                        us += __ldcg(&a.gp[(((int64_t)pc) * g.N + row + 1) * B + tok]);
                    }
                    gemv_final_pair(a, row / 2, tok, gs, us);
                }
            } else {
                for (int u = tid; u < (row1 - row0) * B; u += kGemvThreads) {
                    const int row = row0 + u / B, tok = u % B;
                    SegSums ss;
                    for (int s = 0; s < g.nseg; ++s) {
                        float v = 0.f;
                        for (int pc = 0; pc < g.pieces; ++pc)
                            v += __ldcg(&a.gp[(((int64_t)s * g.pieces + pc) * g.N + row) * B + tok]);
                        ss.p[s] = v;
                    }
                    gemv_final_row(a, row, tok, ss);
                }
            }
            if (tid == 0) atomicExch(&a.tickets[rb], 0u);
        }
    }
    if (tid == 0) {
        TPL_TRACE_AT(3);
        TPL_TRACE_PUT(a.epi == EPI_QKV ? TR_QKV : a.epi == EPI_GU ? TR_GU : a.trace_row_tag);
    }
}

}  // namespace tpl
