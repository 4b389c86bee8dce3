// Decode projections (B <= 64 tokens) on the 5th-generation tensor cores.
//
// D[128 weight rows][NX columns] = W[128][K] . X[NX][K]^T in TMEM, where X
// holds the B tokens' activation rows (bf16; with SPLIT, hi parts in rows
// 0..B-1 and lo parts in rows NX/2..NX/2+B-1, other rows unused; NX =
// 16..128).  For the column-parallel projections X is x * gamma and the
// RMSNorm factor 1/rms is computed by the epilogue warps while the weights
// stream and applied to the results; the row-parallel ones can also write the
// next projection's X from their output.
// The kernel is bound by streaming the weights from HBM: TMA brings 128-row x
// 64-column weight tiles (16 KB, 128-byte swizzle) and the matching activation
// tile into a 4-8 stage shared-memory ring, one thread issues four M=128,
// N=NX, K=16 tcgen05.mma per stage, and the tensor pipe idles most of the
// time.  192 threads: warp 0 TMA producer, warp 1 TMEM owner and MMA issuer,
// warps 2-5 epilogue (one TMEM lane = one weight row each), which walks the
// tokens in chunks of 16 columns so that its registers do not grow with B.
//
// Work division ("stream-K"): the k-blocks of every (row tile, segment) are
// laid end to end, tile-major then segment then k, and each CTA takes one
// contiguous range, so every SM streams the same number of weight bytes.  A
// CTA walks its range in the order of gt_order: the parts of its first and
// last tiles (shared with the neighbouring CTAs) before the tiles in between.
// A run of k-blocks of one (tile, segment) inside a CTA is one MMA chain (a
// "piece").  Segments are the row-parallel shards ("Tensor parallel scaling
// curves", "What tensor parallelism actually splits"); column-parallel
// projections have one.  Order of the sums, fixed for a given SM count:
//   segment sum = pieces in k order;  tile sum = segment sums in shard order.
// A tile whose k-blocks all lie in one CTA is finished in the CTA (running
// sums in shared memory).  A tile
// split across CTAs has each CTA store its pieces to the workspace and add its
// k-block count to the tile's arrival counter; the CTA that completes the
// count adds all pieces in the fixed order (no CTA waits for another) and
// resets the counter.  The fused and separate row-split modes run the same
// pieces and sums, so they agree bit for bit.
//
// Weight tiles for the first stages are requested before the dependency wait
// (programmatic dependent launch): weights never depend on the previous
// kernel.  Every wait is bounded (2 s); a timeout sets the error word, stops
// every role, waits (bounded) for copies in flight and releases TMEM.
#pragma once

#include <cuda.h>

#include "tpl_common.cuh"
#include "tpl_gemm.cuh"

namespace tpl {

constexpr int kGtThreads = 192;
constexpr int kGtRows = 128;     // weight rows per tile (MMA M)
constexpr int kGtK = 64;         // columns per k-block
constexpr int kGtWBytes = kGtRows * kGtK * 2;  // 16 KB
constexpr int kGtBufsMax = 8;    // TMEM accumulators in flight, at most
constexpr int kGtMaxB = 64;       // tokens per call
constexpr int kGtChunk = 16;      // tokens per epilogue chunk
constexpr int kGtList = 120;      // piece list entries per combine chunk
constexpr int kGtBarBytes = 2048;  // mbarriers, flags and the piece lists after the stage ring
constexpr int kGtRmsBytes = 2048;  // per-warp sums of squares and 1/rms per token

// Shared memory: the stage ring, the running tile sums of tiles finished
// inside one CTA ([tokens][128 rows] fp32), then the barrier area.  The ring
// and the tile sums share a 160 KB budget: measured on B200 against 96-208
// KB, a 70B-shaped decode layer ran fastest there (470 us against 551 us at
// 208 KB, with 16 tokens), which leaves the rest of the SM's shared memory to
// the L1 cache and to the next kernel's blocks.
template <int NX, bool SPLIT>
struct GemvTcSmem {
    static constexpr int XBYTES = NX * kGtK * 2;
    static constexpr int STAGE = kGtWBytes + XBYTES;
    static constexpr int TOK = SPLIT ? NX / 2 : NX;  // token columns of the accumulator
    static constexpr int NCH = TOK < kGtChunk ? 1 : TOK / kGtChunk;
    static constexpr int TSBYTES = NCH * kGtChunk * kGtRows * 4;
    static constexpr int NS = (160 * 1024 - TSBYTES) / STAGE;
    // accumulators in flight: as many as TMEM's 512 columns hold, up to 8 (they
    // let the weight stream run on while the epilogue adds split tiles)
    static constexpr int BUFS = 512 / NX < kGtBufsMax ? 512 / NX : kGtBufsMax;
    static constexpr int BYTES = NS * STAGE + TSBYTES + 1024 + kGtBarBytes + kGtRmsBytes;
    static_assert(BYTES <= 232448, "shared memory per block");
};

enum { GT_QKV = 0, GT_GU = 1, GT_ROW = 2, GT_ROW_PARTIAL = 3 };

struct GemvTcArgs {
    CUtensorMap tm_w;   // column ops: 2-D [N][ld]; row ops: 3-D [t][N][ld]
    CUtensorMap tm_x;   // [rows_x][K_x] bf16, box {64, NX}
    int N;              // output rows
    int B;              // tokens
    int tiles, nseg, kbs;  // row tiles, segments per tile, k-blocks per segment
    int64_t U;          // tiles * nseg * kbs
    int x_seg_stride;   // X column offset between segments (row ops), elements
    int w3d;
    int xsplit;         // the activation rows are bf16 hi + lo pairs (the <16, true> kernel serves both forms)
    int epi;
    // outputs
    float *out32;       // GT_ROW
    void *out_act;      // GT_ROW / GT_GU (bf16)
    const void *resid;  // GT_ROW
    int resid_f32;
    float *partials;    // GT_ROW_PARTIAL: [nseg][B][N]
    // QKV scatter (as the matrix-vector kernel)
    float *q;
    float *knew, *vnew;
    __nv_bfloat16 *kc, *vc;
    int rps, nq, nq_s, nkv_s, hd, batch_cap;
    int64_t S, seq_cap;
    // RMSNorm folded in: the activation operand is x * gamma (split_scaled)
    // and the column-op results are multiplied by 1/sqrt(mean(src^2) + eps)
    // per token, computed here from src [B][rms_len] (fp32 or bf16)
    const void *rms_src;
    int rms_f32, rms_len;
    float rms_eps;
    // GT_ROW: also write the next projection's operand from the output
    // (out_act rounded when present): xs_out rows b (hi) and xs_half + b (lo)
    __nv_bfloat16 *xs_out;
    const float *xs_gamma;
    int xs_half;
    // cross-CTA pieces and arrival counters
    float *gpart;       // [G][2][nseg][gstride / 4][128] float4: token quads outer, rows inner
    int gstride;        // floats per row of a piece: 16 * ceil(B / 16)
    unsigned *tickets;  // [tiles]
    int trace_row_tag;  // timeline tag of a row-parallel launch (traced builds)
};

// Tokens 16*ch .. 16*ch+15 of one accumulator row: the hi column plus the
// lo column NX/2 further (SPLIT), or the column itself.  With 16 columns and
// at most 8 tokens the two forms share one shared-memory layout, so one
// kernel serves the split and the unsplit projections (xsplit chooses at run
// time): the four projections of a layer then run the same code, and the
// end-of-kernel code one of them fetched into the instruction cache is still
// there for the next (stack layer 317 -> 315 us).
template <int NX, bool SPLIT>
__device__ __forceinline__ void gt_load_chunk(uint32_t taddr, int ch, float (&pv)[kGtChunk], bool xsplit) {
    if constexpr (SPLIT && NX == 16) {
        if (xsplit) {  // 8 tokens: hi in columns 0..7, lo in 8..15
            float d[16];
            tmem_ld16(taddr, d);
#pragma unroll
            for (int t = 0; t < 16; ++t) pv[t] = t < 8 ? d[t] + d[8 + t] : 0.f;
        } else {
            tmem_ld16(taddr, pv);
        }
    } else if constexpr (SPLIT) {
        if (xsplit) {
            float hi[16], lo[16];
            tmem_ld16(taddr + (uint32_t)(16 * ch), hi);
            tmem_ld16(taddr + (uint32_t)(NX / 2 + 16 * ch), lo);
#pragma unroll
            for (int t = 0; t < 16; ++t) pv[t] = hi[t] + lo[t];
        } else {  // unsplit tokens in the first NX/2 columns, the rest zero
            tmem_ld16(taddr + (uint32_t)(16 * ch), pv);
        }
    } else {
        tmem_ld16(taddr + (uint32_t)(16 * ch), pv);
    }
}

// CTA c's unit range [u0, u1) of U units over G CTAs.
__device__ __forceinline__ int64_t gt_start(int64_t U, int G, int c) {
    // 32-bit arithmetic when it cannot overflow (c <= G <= 256): much cheaper
    // than a 64-bit division, and the combine evaluates this many times
    if (U < (1ll << 23)) return (int64_t)(((uint32_t)U * (uint32_t)c) / (uint32_t)G);
    return U * c / G;
}

// The order in which a CTA walks its range, as three sub-ranges [b, e): the
// part of its first tile, the part of its last tile (both possibly shared
// with the neighbouring CTAs), then the whole tiles in between.  Taking the
// shared parts first lets the CTA that completes a shared tile add its pieces
// early, while its own weight stream continues, instead of at the end of the
// kernel (where that combine measured 10-20 us of the critical path).
struct GtOrder {
    int64_t u0, u1, f_end, l_beg;
    // sub-range s: [0] = [u0, f_end), [1] = [l_beg, u1), [2] = [f_end, l_beg)
    __device__ __forceinline__ int64_t b(int s) const { return s == 0 ? u0 : (s == 1 ? l_beg : f_end); }
    __device__ __forceinline__ int64_t e(int s) const { return s == 0 ? f_end : (s == 1 ? u1 : l_beg); }
};
__device__ __forceinline__ GtOrder gt_order(int64_t u0, int64_t u1, int64_t per_tile) {
    GtOrder o;
    o.u0 = u0;
    o.u1 = u1;
    o.f_end = min(u1, (u0 / per_tile + 1) * per_tile);
    o.l_beg = max(o.f_end, ((u1 - 1) / per_tile) * per_tile);
    return o;
}

// Final write of one output row for tokens tok0 .. tok0+15 (fused sums or
// column ops).  This and gt_combine run at the end of the kernel, once per
// CTA, where their code is cold (fetched from L2 line by line, which measured
// several us): both are kept short -- per-row destinations computed once, a
// few stores per token, the piece list built in parallel.  (Non-inlined
// copies, and a spare warp running them early to warm the instruction cache,
// both measured slower.)
// The loads the row-parallel final write needs (the residual of the chunk's
// tokens and the row's gain for the next operand), issued early so that
// their latency overlaps the combine's own loads.
struct GtRowIn {
    float rv[kGtChunk];
    float gam;
};
// Per-token code of the end-of-kernel writes runs for the chunk's first 4
// tokens, and for the other 12 only behind one branch taken when the chunk
// holds more: at 4 tokens or fewer the 12 copies are never fetched, which
// matters for code that runs cold (about 1.5 us of the row-parallel combine).
template <typename F>
__device__ __forceinline__ void gt_for_tokens(int ntok, F &&f) {
#pragma unroll
    for (int j = 0; j < 4; ++j) f(j);
    if (ntok > 4) {
#pragma unroll
        for (int j = 4; j < kGtChunk; ++j) f(j);
    }
}

__device__ __forceinline__ void gt_row_loads(const GemvTcArgs &a, int row, int tok0, GtRowIn &in) {
    const int B = a.B;
    const bool ok = row < a.N && a.resid;
    const int64_t base = (int64_t)tok0 * a.N + row;
    if (a.resid_f32) {
        const float *r = static_cast<const float *>(a.resid) + base;
        gt_for_tokens(B - tok0, [&](int j) { in.rv[j] = (ok && tok0 + j < B) ? r[(int64_t)j * a.N] : 0.f; });
    } else {
        const __nv_bfloat16 *r = static_cast<const __nv_bfloat16 *>(a.resid) + base;
        gt_for_tokens(B - tok0, [&](int j) {
            in.rv[j] = (ok && tok0 + j < B) ? __bfloat162float(r[(int64_t)j * a.N]) : 0.f;
        });
    }
    in.gam = (row < a.N && a.xs_gamma) ? a.xs_gamma[row] : 1.f;
}

__device__ __forceinline__ void gt_final(const GemvTcArgs &a, int row, const float (&v0)[kGtChunk], int lane, int tok0,
                                      const float *inv_rms, const GtRowIn *pre = nullptr) {
    const int B = a.B;
    const bool scale = a.rms_src && a.epi != GT_ROW;  // the RMSNorm factor of column ops
    const int ntok = B - tok0;
    float v[kGtChunk];
    gt_for_tokens(ntok, [&](int i) { v[i] = scale ? v0[i] * inv_rms[min(tok0 + i, kGtMaxB - 1)] : v0[i]; });
    if (a.epi == GT_GU) {
        // rows interleave gate and up: the even lane pairs with its odd neighbour
        const bool w = !(lane & 1) && row + 1 < a.N;
        __nv_bfloat16 *dst = static_cast<__nv_bfloat16 *>(a.out_act) + row / 2;
        const int64_t st = a.N / 2;
        gt_for_tokens(ntok, [&](int i) {
            const int b = tok0 + i;
            const float u = __shfl_down_sync(0xffffffffu, v[i], 1);
            if (w && b < B) dst[b * st] = __float2bfloat16_rn(silu(v[i]) * u);
        });
        return;
    }
    if (row >= a.N) return;
    if (a.epi == GT_QKV) {
        // the row is one q element, or one k or v element of the cache (and
        // its fp32 copy); per token only the batch stride moves
        const int s = row / a.rps, l = row % a.rps;
        const int qd = a.nq_s * a.hd, kd = a.nkv_s * a.hd;
        const bool isq = l < qd;
        const bool isk = l < qd + kd;
        const int ll = isk ? l - qd : l - qd - kd;  // kv head * hd + dim within the shard
        float *dq = a.q + (int64_t)s * qd + l;
        __nv_bfloat16 *dc = (isk ? a.kc : a.vc) + ((int64_t)s * a.batch_cap * a.nkv_s * a.seq_cap + a.S) * a.hd +
                            (int64_t)(ll / a.hd) * a.seq_cap * a.hd + ll % a.hd;
        float *dn = isk ? a.knew : a.vnew;
        if (dn) dn += (int64_t)s * kd + ll;
        const int64_t sq = (int64_t)a.nq * a.hd, sc = (int64_t)a.nkv_s * a.seq_cap * a.hd,
                      sn = (int64_t)a.nkv_s * (a.nq / a.nq_s) * a.hd;
        gt_for_tokens(ntok, [&](int i) {
            const int b = tok0 + i;
            if (b >= B) return;
            if (isq) {
                dq[b * sq] = v[i];
            } else {
                dc[b * sc] = __float2bfloat16_rn(v[i]);
                if (dn) dn[b * sn] = v[i];
            }
        });
        return;
    }
    // GT_ROW: out = resid + sum.  Every load before any store (the pointers
    // may alias as far as the compiler knows, which would otherwise
    // serialise the loads' latencies); the combine issues them even earlier.
    GtRowIn in_local;
    if (!pre) gt_row_loads(a, row, tok0, in_local);
    const GtRowIn &in = pre ? *pre : in_local;
    const float *rv = in.rv;
    const float gam = in.gam;
    __nv_bfloat16 *oact = static_cast<__nv_bfloat16 *>(a.out_act);
    gt_for_tokens(ntok, [&](int j) {
        const int b = tok0 + j;
        if (b >= B) return;
        const int64_t i = (int64_t)b * a.N + row;
        const float o = a.resid ? rv[j] + v[j] : v[j];
        if (a.out32) a.out32[i] = o;
        if (oact) oact[i] = __float2bfloat16_rn(o);
        if (a.xs_out) {
            // the next projection's operand: split_scaled with the row's gain loaded once
            const float src = oact ? __bfloat162float(__float2bfloat16_rn(o)) : o;
            const float sc = a.xs_gamma ? __fmul_rn(src, gam) : src;
            const __nv_bfloat16 hi = __float2bfloat16_rn(sc);
            a.xs_out[i] = hi;
            a.xs_out[(int64_t)(a.xs_half + b) * a.N + row] = __float2bfloat16_rn(__fsub_rn(sc, __bfloat162float(hi)));
        }
    });
}

// The CTA that completed a tile split across CTAs adds its pieces in the
// fixed order (segment, then CTA) and writes the tile.  The CTAs cf..cl cover
// the tile; with at most 128 (segment, CTA) candidates the 128 epilogue
// threads test one each and compact the list in candidate order, else one
// thread generates it in rounds of up to kGtList entries.  The pieces are
// then loaded (with at most 4 tokens in the chunk one float4 each, 16 in
// flight; else 8 pieces of 4 float4) and added in list order; the walk is
// repeated for each 16-token chunk, reusing the list when one round held it
// all.  Each CTA stored its part in slot 0 if the tile is its first, else in
// slot 1.  Run by the 128 epilogue threads (named barrier 1).
// The CTAs cf..cl whose unit ranges cover a tile.
__device__ __forceinline__ void gt_tile_ctas(const GemvTcArgs &a, int tile, int G, int &cf, int &cl) {
    const int64_t per_tile = (int64_t)a.nseg * a.kbs;
    const int64_t t_beg = (int64_t)tile * per_tile;
    cf = (int)((t_beg * G) / a.U);
    while (cf > 0 && gt_start(a.U, G, cf) > t_beg) --cf;
    while (gt_start(a.U, G, cf + 1) <= t_beg) ++cf;
    cl = cf;
    while (cl + 1 < G && gt_start(a.U, G, cl + 1) < t_beg + per_tile) ++cl;
}

// A split tile's piece list in the fixed order (segment, then CTA) built by
// the 128 epilogue threads at once: with at most 128 (segment, CTA)
// candidates each thread tests one and the valid ones are compacted by ballot
// into list[0, *nlist).  Returns whether the whole list was built (false:
// too many candidates, or a full list that may have dropped entries).  All
// 128 threads call it (named barrier 1); cnt is scratch for 4 counts.
__device__ __forceinline__ bool gt_build_list(const GemvTcArgs &a, int tile, int G, int lane, int ep_tid,
                                           volatile int *list, volatile int *nlist, volatile int *cnt) {
    const int64_t per_tile = (int64_t)a.nseg * a.kbs;
    const int64_t t_beg = (int64_t)tile * per_tile;
    int cf, cl;
    gt_tile_ctas(a, tile, G, cf, cl);
    const int ncta = cl - cf + 1, ncand = a.nseg * ncta;
    if (ncand > 128) return false;
    const int g_s = ep_tid / ncta, c = cf + ep_tid % ncta;
    bool valid = false;
    int ent = 0;
    if (ep_tid < ncand) {
        const int64_t sb = t_beg + (int64_t)g_s * a.kbs, se = sb + a.kbs;
        const int64_t c0 = gt_start(a.U, G, c), c1 = gt_start(a.U, G, c + 1);
        valid = c1 > sb && c0 < se;
        const int sl = (tile == (int)(c0 / per_tile)) ? 0 : 1;
        ent = (((c * 2 + sl) * a.nseg + g_s) << 5) | (g_s << 1) | (c1 >= se ? 1 : 0);
    }
    const unsigned m = __ballot_sync(0xffffffffu, valid);
    const int w = ep_tid >> 5;
    if (lane == 0) cnt[w] = __popc(m);
    asm volatile("bar.sync 1, 128;" ::: "memory");
    int base = 0;
    for (int x = 0; x < w; ++x) base += cnt[x];
    const int pos = base + __popc(m & ((1u << lane) - 1u));
    if (valid && pos < kGtList) list[pos] = ent;
    const int tot = cnt[0] + cnt[1] + cnt[2] + cnt[3];
    if (ep_tid == 0) *nlist = tot < kGtList ? tot : kGtList;
    asm volatile("bar.sync 1, 128;" ::: "memory");
    return tot < kGtList;
}

// `pre`/`pre_n`: the tile's piece list built while the weights streamed
// (pre_n < 0: none), which spares the combine, run cold at the end of the
// kernel, the candidate search.
__device__ __forceinline__ void gt_combine(const GemvTcArgs &a, int tile, int G, int nch, int r, int lane, int ep_tid,
                                        const float *s_inv, volatile int *s_list, volatile int *s_nlist,
                                        volatile int *s_more, volatile int *s_cnt, const volatile int *pre,
                                        int pre_n) {
    const int64_t per_tile = (int64_t)a.nseg * a.kbs;
    const int64_t t_beg = (int64_t)tile * per_tile;
    const int row = tile * kGtRows + r;
    const int B = a.B;
    float seg_sum[kGtChunk], tile_sum[kGtChunk];
    GtRowIn row_in;                  // the row-parallel final write's loads, issued with the pieces'
    bool single = pre_n >= 0;        // the whole list is in shared memory
    const volatile int *lst = single ? pre : s_list;
#ifdef TPL_TRACE
    // SM-clock marks of the first chunk (traced builds): start, list built,
    // pieces loaded and added, written
    uint64_t ck[4] = {(uint64_t)clock64(), 0, 0, 0};
#endif
#pragma unroll 1
    for (int ch = 0; ch < nch; ++ch) {
        const int tok0 = kGtChunk * ch;
#pragma unroll
        for (int t = 0; t < kGtChunk; ++t) {
            tile_sum[t] = -0.f;
            seg_sum[t] = -0.f;
        }
        int g_s = 0, g_cc = 0;  // generator position (thread 0)
        if (!single) {
            single = gt_build_list(a, tile, G, lane, ep_tid, s_list, s_nlist, s_cnt);
            if (ep_tid == 0) *s_more = 0;
            int cl;
            gt_tile_ctas(a, tile, G, g_cc, cl);
        }
        for (int round = 0;; ++round) {
            if (!single) {
                if (ep_tid == 0) {
                    int n = 0;
                    while (n < kGtList && g_s < a.nseg) {
                        const int64_t sb = t_beg + (int64_t)g_s * a.kbs, se = sb + a.kbs;
                        const int64_t c0 = gt_start(a.U, G, g_cc), c1 = gt_start(a.U, G, g_cc + 1);
                        if (c1 > sb && c0 < se) {
                            const int sl = (tile == (int)(c0 / per_tile)) ? 0 : 1;
                            const bool seg_last = c1 >= se;
                            s_list[n++] = (((g_cc * 2 + sl) * a.nseg + g_s) << 5) | (g_s << 1) | (seg_last ? 1 : 0);
                        }
                        if (c1 >= se) {
                            ++g_s;  // next segment starts in this same CTA
                        } else {
                            ++g_cc;
                        }
                    }
                    *s_nlist = n;
                    *s_more = g_s < a.nseg ? 1 : 0;
                }
                asm volatile("bar.sync 1, 128;" ::: "memory");
            }
            const int n = lst == pre ? pre_n : *s_nlist;
#ifdef TPL_TRACE
            if (ch == 0 && round == 0) ck[1] = (uint64_t)clock64();
#endif
            auto piece_src = [&](int ent) {
                return reinterpret_cast<const float4 *>(a.gpart) +
                       ((int64_t)(ent >> 5) * (a.gstride / 4) + tok0 / 4) * kGtRows + r;
            };
            if (a.epi == GT_ROW && round == 0) gt_row_loads(a, row, tok0, row_in);
            if (B - tok0 <= 4) {
                float4 seg4 = make_float4(seg_sum[0], seg_sum[1], seg_sum[2], seg_sum[3]);
                float4 tile4 = make_float4(tile_sum[0], tile_sum[1], tile_sum[2], tile_sum[3]);
                for (int e0 = 0; e0 < n; e0 += 16) {
                    float4 v1[16];
                    int en[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        en[j] = e0 + j < n ? lst[e0 + j] : 0;
                        v1[j] = e0 + j < n ? __ldcg(piece_src(en[j])) : make_float4(0.f, 0.f, 0.f, 0.f);
                    }
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        if (e0 + j >= n) break;
                        seg4.x = seg4.x + v1[j].x;
                        seg4.y = seg4.y + v1[j].y;
                        seg4.z = seg4.z + v1[j].z;
                        seg4.w = seg4.w + v1[j].w;
                        if (en[j] & 1) {  // the segment is complete
                            if (a.epi == GT_ROW_PARTIAL) {
                                if (row < a.N) {
                                    const int sg = (en[j] >> 1) & 15;
                                    float *dst = a.partials + ((int64_t)sg * B + tok0) * a.N + row;
                                    const float w4[4] = {seg4.x, seg4.y, seg4.z, seg4.w};
#pragma unroll
                                    for (int t = 0; t < 4; ++t)
                                        if (tok0 + t < B) dst[t * a.N] = w4[t];
                                }
                            } else {
                                tile4.x = tile4.x + seg4.x;
                                tile4.y = tile4.y + seg4.y;
                                tile4.z = tile4.z + seg4.z;
                                tile4.w = tile4.w + seg4.w;
                            }
                            seg4 = make_float4(-0.f, -0.f, -0.f, -0.f);
                        }
                    }
                }
                seg_sum[0] = seg4.x;
                seg_sum[1] = seg4.y;
                seg_sum[2] = seg4.z;
                seg_sum[3] = seg4.w;
                tile_sum[0] = tile4.x;
                tile_sum[1] = tile4.y;
                tile_sum[2] = tile4.z;
                tile_sum[3] = tile4.w;
            } else {
                for (int e0 = 0; e0 < n; e0 += 8) {
                    float4 v[8][kGtChunk / 4];
                    int en[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        en[j] = e0 + j < n ? lst[e0 + j] : 0;
                        const float4 *src = piece_src(en[j]);
#pragma unroll
                        for (int q4 = 0; q4 < kGtChunk / 4; ++q4)
                            v[j][q4] = (e0 + j < n && tok0 + 4 * q4 < B) ? __ldcg(src + q4 * kGtRows)
                                                                        : make_float4(0.f, 0.f, 0.f, 0.f);
                    }
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        if (e0 + j >= n) break;
#pragma unroll
                        for (int q4 = 0; q4 < kGtChunk / 4; ++q4) {
                            seg_sum[4 * q4] = seg_sum[4 * q4] + v[j][q4].x;
                            seg_sum[4 * q4 + 1] = seg_sum[4 * q4 + 1] + v[j][q4].y;
                            seg_sum[4 * q4 + 2] = seg_sum[4 * q4 + 2] + v[j][q4].z;
                            seg_sum[4 * q4 + 3] = seg_sum[4 * q4 + 3] + v[j][q4].w;
                        }
                        if (en[j] & 1) {  // the segment is complete
                            const int sg = (en[j] >> 1) & 15;
                            if (a.epi == GT_ROW_PARTIAL) {
                                if (row < a.N) {
                                    float *dst = a.partials + ((int64_t)sg * B + tok0) * a.N + row;
#pragma unroll
                                    for (int t = 0; t < kGtChunk; ++t)
                                        if (tok0 + t < B) dst[t * a.N] = seg_sum[t];
                                }
                            } else {
#pragma unroll
                                for (int t = 0; t < kGtChunk; ++t) tile_sum[t] = tile_sum[t] + seg_sum[t];
                            }
#pragma unroll
                            for (int t = 0; t < kGtChunk; ++t) seg_sum[t] = -0.f;
                        }
                    }
                }
            }
#ifdef TPL_TRACE
            if (ch == 0 && round == 0) ck[2] = (uint64_t)clock64();
#endif
            if (single) break;
            const bool more = *s_more != 0;
            asm volatile("bar.sync 1, 128;" ::: "memory");  // list consumed before it is rewritten
            if (!more) {
                single = round == 0;  // one round held the whole list: keep it
                break;
            }
        }
        if (a.epi != GT_ROW_PARTIAL) gt_final(a, row, tile_sum, lane, tok0, s_inv, a.epi == GT_ROW ? &row_in : nullptr);
#ifdef TPL_TRACE
        if (ch == 0) {
            ck[3] = (uint64_t)clock64();
            if (ep_tid == 0)
                trace_put(200 + (a.epi == GT_QKV ? TR_QKV : a.epi == GT_GU ? TR_GU : a.trace_row_tag), ck);
        }
#endif
    }
}

template <int NX, bool SPLIT>
__global__ void __launch_bounds__(kGtThreads, 1) gemv_tc_kernel(const __grid_constant__ GemvTcArgs a) {
    using SMEM = GemvTcSmem<NX, SPLIT>;
    constexpr int STAGE = SMEM::STAGE;
    constexpr int NS = SMEM::NS;
    constexpr int BUFS = SMEM::BUFS;
    static_assert(2 * NS * 8 + 2 * BUFS * 8 + 8 + 4 + 32 + 4 * (kGtList + 4) + 4 * (2 * kGtList + 2) <= kGtBarBytes,
                  "barrier area");
    constexpr int TMEM_COLS = BUFS * NX <= 32 ? 32 : BUFS * NX <= 64 ? 64 : BUFS * NX <= 128 ? 128
                              : BUFS * NX <= 256 ? 256 : 512;
    static_assert(BUFS * NX <= 512, "accumulators");
    extern __shared__ __align__(1024) unsigned char gv_raw[];
    unsigned char *sm = reinterpret_cast<unsigned char *>(((uintptr_t)gv_raw + 1023) & ~(uintptr_t)1023);
    float *ts = reinterpret_cast<float *>(sm + NS * STAGE);  // [NCH * 16 tokens][128 rows]
    uint64_t *full = reinterpret_cast<uint64_t *>(sm + NS * STAGE + SMEM::TSBYTES);
    float *s_rpart = reinterpret_cast<float *>(sm + NS * STAGE + SMEM::TSBYTES + kGtBarBytes);  // [4][kGtMaxB]
    float *s_inv = s_rpart + 4 * kGtMaxB;                                                       // [kGtMaxB]
    static_assert(5 * kGtMaxB * 4 <= kGtRmsBytes, "rms area");
    uint64_t *empty = full + NS;
    uint64_t *acc_full = empty + NS;        // [BUFS]
    uint64_t *acc_empty = acc_full + BUFS;  // [BUFS]
    uint64_t *fin = acc_empty + BUFS;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(fin + 1);
    volatile int *s_fail = reinterpret_cast<volatile int *>(tmem_slot + 1);
    int *s_issued = const_cast<int *>(s_fail) + 1;
    int *s_consumed = const_cast<int *>(s_fail) + 2;
    volatile int *s_last = const_cast<int *>(s_fail) + 3;
    volatile int *s_nlist = const_cast<int *>(s_fail) + 4;
    volatile int *s_more = const_cast<int *>(s_fail) + 5;
    volatile int *s_list = const_cast<int *>(s_fail) + 8;  // [kGtList]
    volatile int *s_pre = s_list + kGtList + 4;              // [2][kGtList]: lists of the first and last tile
    volatile int *s_pre_n = s_pre + 2 * kGtList;             // [2]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = gridDim.x, cta = blockIdx.x;
    const int64_t u0 = gt_start(a.U, G, cta), u1 = gt_start(a.U, G, cta + 1);
    const int64_t per_tile = (int64_t)a.nseg * a.kbs;
    TPL_TRACE_VARS
    if (threadIdx.x == 0) TPL_TRACE_AT(0);

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < BUFS; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 4);
        }
        mbar_init(fin, 1);
        *s_fail = 0;
        *s_issued = 0;
        *s_consumed = 0;
        *s_last = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(TMEM_COLS));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = *tmem_slot;
    // every thread lets the next kernel be scheduled; only what this kernel
    // reads from earlier kernels (the activations) waits for them
    pdl_trigger();

    if (warp == 0) {
        if (lane == 0) {
            // (tile, segment, k-block) of each unit in the walking order:
            // located by division at the start of a sub-range, then stepped
            const GtOrder ord = gt_order(u0, u1, per_tile);
            int sr = 0, tile = 0, seg = 0, kb = 0;
            int64_t uu = u0;
            auto locate = [&]() {
                tile = (int)(uu / per_tile);
                const int w = (int)(uu - (int64_t)tile * per_tile);
                seg = w / a.kbs;
                kb = w - seg * a.kbs;
            };
            auto restart = [&]() {
                sr = 0;
                uu = ord.b(0);
                locate();
            };
            auto advance = [&]() {
                if (++uu < ord.e(sr)) {
                    if (++kb == a.kbs) {
                        kb = 0;
                        if (++seg == a.nseg) {
                            seg = 0;
                            ++tile;
                        }
                    }
                    return;
                }
                while (++sr < 3 && ord.b(sr) >= ord.e(sr)) {
                }
                if (sr < 3) {
                    uu = ord.b(sr);
                    locate();
                }
            };
            const int n = (int)(u1 - u0);
            const int pre = n < NS ? n : NS;
            const uint64_t wpol = evict_first_policy();  // the weights are read once
            // weight tiles of the first stages before the dependency wait
            // (weights never depend on the previous kernel)
            restart();
            for (int i = 0; i < pre; ++i, advance()) {
                unsigned char *st = sm + i * STAGE;
                mbar_expect_tx(&full[i], STAGE);
                if (a.w3d) tma_load_3d_hint(st, &a.tm_w, kb * kGtK, tile * kGtRows, seg, &full[i], wpol);
                else tma_load_2d_hint(st, &a.tm_w, kb * kGtK, tile * kGtRows, &full[i], wpol);
            }
            pdl_wait();
            TPL_TRACE_AT(1);
            restart();
            int it = 0;
            for (; it < n; ++it, advance()) {
                const int s = it % NS;
                unsigned char *st = sm + s * STAGE;
                if (it >= pre) {
                    const unsigned ph = (unsigned)(it / NS) & 1u;
                    if (*s_fail || !mbar_wait(&empty[s], ph ^ 1u)) {
                        *s_fail = 1;
                        break;
                    }
                    mbar_expect_tx(&full[s], STAGE);
                    if (a.w3d) tma_load_3d_hint(st, &a.tm_w, kb * kGtK, tile * kGtRows, seg, &full[s], wpol);
                    else tma_load_2d_hint(st, &a.tm_w, kb * kGtK, tile * kGtRows, &full[s], wpol);
                }
                tma_load_2d(st + kGtWBytes, &a.tm_x, seg * a.x_seg_stride + kb * kGtK, 0, &full[s]);
            }
            *s_issued = it;
            TPL_TRACE_AT(2);
        }
    } else if (warp == 1) {
        pdl_wait();
        if (lane == 0) {
            constexpr uint32_t IDESC = umma_idesc(kGtRows, NX);
            const GtOrder ord = gt_order(u0, u1, per_tile);
            int it = 0, c = 0;
            bool ok = true;
            for (int sr = 0; ok && sr < 3; ++sr)
            for (int64_t u = ord.b(sr); ok && u < ord.e(sr); ++c) {
                // one piece: the run of k-blocks of one (tile, segment)
                const int64_t seg_end = (u / a.kbs + 1) * a.kbs;  // segments are kbs-aligned in u
                const int64_t pe = min(ord.e(sr), seg_end);
                const int b = c % BUFS;
                const unsigned use = (unsigned)(c / BUFS);
                if (*s_fail || !mbar_wait(&acc_empty[b], (use & 1u) ^ 1u)) {
                    ok = false;
                    break;
                }
                asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                const uint32_t d = tmem + (uint32_t)(b * NX);
                for (int64_t v = u; v < pe; ++v, ++it) {
                    const int s = it % NS;
                    if (*s_fail || !mbar_wait(&full[s], (unsigned)(it / NS) & 1u)) {
                        ok = false;
                        break;
                    }
                    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                    const unsigned sw = smem_u32(sm + s * STAGE);
                    const unsigned sx = sw + kGtWBytes;
#pragma unroll
                    for (int k = 0; k < kGtK / 16; ++k)
                        umma(d, umma_desc(sw + 32 * k), umma_desc(sx + 32 * k), IDESC, (v > u || k > 0) ? 1u : 0u);
                    umma_commit(&empty[s]);
                }
                if (!ok) break;
                umma_commit(&acc_full[b]);
                u = pe;
            }
            if (!ok) *s_fail = 1;
            *s_consumed = it;
            umma_commit(fin);
            if (!mbar_wait(fin, 0)) *s_fail = 1;
        }
    } else {
        pdl_wait();
        // ---- epilogue: thread = weight row 32*(warp%4) + lane of the tile ----
        // A warp whose wait runs out keeps walking the same pieces with the
        // work suppressed (`dead`), so the named barriers below still meet.
        // Tokens are handled in chunks of 16 columns (nch of them).
        const int q = warp & 3;
        const int r = 32 * q + lane;
        const uint32_t lane_off = (uint32_t)(32 * q) << 16;
        const int B = a.B;
        const int nch = min((B + kGtChunk - 1) / kGtChunk, SMEM::NCH);
        const int ep_tid = threadIdx.x - 64;  // 0..127
        // epilogue marks of the last shared tile (traced builds): pieces
        // published, arrival counted, pieces listed, tile finished
        TPL_TRACE_VARS
        bool ep_traced = false;
        if (a.rms_src) {
            // 1/rms per token while the first weight tiles stream in: each
            // warp sums the squares of a strided quarter of the row, the four
            // quarters are added in a fixed order
            const int n8 = a.rms_len / 8;
            for (int b = 0; b < B; ++b) {
                float ss = 0.f;
                for (int c8 = ep_tid; c8 < n8; c8 += 128) {
                    float v[8];
                    if (a.rms_f32) {
                        const float4 *p4 = reinterpret_cast<const float4 *>(static_cast<const float *>(a.rms_src) +
                                                                            (int64_t)b * a.rms_len + 8 * c8);
                        const float4 u0 = p4[0], u1 = p4[1];
                        v[0] = u0.x; v[1] = u0.y; v[2] = u0.z; v[3] = u0.w;
                        v[4] = u1.x; v[5] = u1.y; v[6] = u1.z; v[7] = u1.w;
                    } else {
                        const uint4 u = *reinterpret_cast<const uint4 *>(
                            static_cast<const __nv_bfloat16 *>(a.rms_src) + (int64_t)b * a.rms_len + 8 * c8);
                        const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            v[2 * e] = bf16lo(w4[e]);
                            v[2 * e + 1] = bf16hi(w4[e]);
                        }
                    }
#pragma unroll
                    for (int e = 0; e < 8; ++e) ss = fmaf(v[e], v[e], ss);
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
                if (lane == 0) s_rpart[(ep_tid >> 5) * kGtMaxB + b] = ss;
            }
            asm volatile("bar.sync 1, 128;" ::: "memory");
            if (ep_tid < B) {
                const float tot = ((s_rpart[ep_tid] + s_rpart[kGtMaxB + ep_tid]) + s_rpart[2 * kGtMaxB + ep_tid]) +
                                  s_rpart[3 * kGtMaxB + ep_tid];
                s_inv[ep_tid] = 1.0f / sqrtf(tot / (float)a.rms_len + a.rms_eps);
            }
            asm volatile("bar.sync 1, 128;" ::: "memory");
        }
        // the piece lists of this CTA's first and last tiles where other CTAs
        // share them, built now while the weights stream: the CTA that
        // completes such a tile combines it at the end of the kernel, cold
        int pre_tile[2] = {-1, -1};
        if (u1 > u0) {
#pragma unroll 1
            for (int k = 0; k < 2; ++k) {
                const int tl = (int)((k ? u1 - 1 : u0) / per_tile);
                const int64_t tb = (int64_t)tl * per_tile;
                if ((k == 1 && tl == pre_tile[0]) || (tb >= u0 && tb + per_tile <= u1)) continue;
                if (gt_build_list(a, tl, G, lane, ep_tid, s_pre + k * kGtList, s_pre_n + k, s_list + kGtList))
                    pre_tile[k] = tl;
            }
        }
        float tile_sum[kGtChunk];
        int c = 0;
        bool dead = false;
        const GtOrder ord = gt_order(u0, u1, per_tile);
        for (int sr = 0; sr < 3; ++sr)
        for (int64_t u = ord.b(sr); u < ord.e(sr);) {
            const int tile = (int)(u / per_tile);
            const int64_t t_beg = (int64_t)tile * per_tile, t_end = t_beg + per_tile;
            const bool local = t_beg >= u0 && t_end <= u1;
            const int slot = (tile == (int)(u0 / per_tile)) ? 0 : 1;
            const int64_t stop = min(ord.e(sr), t_end);  // this CTA's part of the tile: one sub-range holds all of it
            while (u < stop) {
                const int seg = (int)((u % per_tile) / a.kbs);
                const int64_t pe = min(stop, (u / a.kbs + 1) * a.kbs);
                const int b = c % BUFS;
                ++c;
                u = pe;
                if (!dead)
                    dead = !__all_sync(0xffffffffu,
                                       !*s_fail && mbar_wait(&acc_full[b], (unsigned)((c - 1) / BUFS) & 1u));
                if (dead) {
                    *s_fail = 1;
                    continue;
                }
                asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                const uint32_t acc = tmem + lane_off + (uint32_t)(b * NX);
#pragma unroll 1
                for (int ch = 0; ch < nch; ++ch) {
                    // tokens 16*ch + t: hi part in column 16*ch + t, lo part NX/2 further
                    float pv[kGtChunk];
                    gt_load_chunk<NX, SPLIT>(acc, ch, pv, a.xsplit != 0);
                    if (local) {
                        // every segment of a tile inside this CTA is one piece;
                        // -0 is the additive identity, so segment 0 is stored unchanged
                        float *tsp = ts + (kGtChunk * ch) * kGtRows + r;
#pragma unroll
                        for (int t = 0; t < kGtChunk; ++t)
                            tsp[t * kGtRows] = (seg == 0 ? -0.f : tsp[t * kGtRows]) + pv[t];
                        if (a.epi == GT_ROW_PARTIAL) {
                            const int row = tile * kGtRows + r;
                            if (row < a.N)
#pragma unroll
                                for (int t = 0; t < kGtChunk; ++t)
                                    if (kGtChunk * ch + t < B)
                                        a.partials[((int64_t)seg * B + kGtChunk * ch + t) * a.N + row] = pv[t];
                        }
                    } else {
                        // float4 of tokens 4j..4j+3 of all 128 rows side by side:
                        // a warp's stores cover 512 contiguous bytes
                        float4 *dst = reinterpret_cast<float4 *>(a.gpart) +
                                      ((((int64_t)cta * 2 + slot) * a.nseg + seg) * (a.gstride / 4) + 4 * ch) * kGtRows +
                                      r;
#pragma unroll
                        for (int t = 0; t < kGtChunk; t += 4)
                            if (kGtChunk * ch + t < B)
                                dst[(t / 4) * kGtRows] = make_float4(pv[t], pv[t + 1], pv[t + 2], pv[t + 3]);
                    }
                }
                asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
                __syncwarp();
                if (lane == 0) mbar_arrive(&acc_empty[b]);
            }
            const int row = tile * kGtRows + r;
            if (local) {
                if (!dead && a.epi != GT_ROW_PARTIAL) {
#pragma unroll 1
                    for (int ch = 0; ch < nch; ++ch) {
                        const float *tsp = ts + (kGtChunk * ch) * kGtRows + r;
#pragma unroll
                        for (int t = 0; t < kGtChunk; ++t) tile_sum[t] = tsp[t * kGtRows];
                        gt_final(a, row, tile_sum, lane, kGtChunk * ch, s_inv);
                    }
                }
                continue;
            }
            // shared tile: publish the pieces; the CTA completing the tile adds them
            if (ep_tid == 0) {
                TPL_TRACE_AT(0);
                TPL_TRACE_AT(1);
                TPL_TRACE_AT(2);
                TPL_TRACE_AT(3);
                ep_traced = true;
            }
            __threadfence();
            asm volatile("bar.sync 1, 128;" ::: "memory");
            if (ep_tid == 0) {
                bool last = false;
                if (!*s_fail) {
                    const unsigned mine = (unsigned)(min(u1, t_end) - max(u0, t_beg));
                    const unsigned prev = atomicAdd(&a.tickets[tile], mine);
                    last = prev + mine == (unsigned)per_tile;
                    if (prev + mine > (unsigned)per_tile) record_error(16u);
                    if (last) atomicExch(&a.tickets[tile], 0u);
                }
                *s_last = last ? 1 : 0;
                TPL_TRACE_AT(1);
                TPL_TRACE_AT(2);
                TPL_TRACE_AT(3);
            }
            asm volatile("bar.sync 1, 128;" ::: "memory");
            if (!*s_last) continue;
            __threadfence();
            const int pk = tile == pre_tile[0] ? 0 : tile == pre_tile[1] ? 1 : -1;
            gt_combine(a, tile, G, nch, r, lane, ep_tid, s_inv, s_list, s_nlist, s_more, s_list + kGtList,
                       pk >= 0 ? s_pre + pk * kGtList : nullptr, pk >= 0 ? s_pre_n[pk] : -1);
            if (ep_tid == 0) TPL_TRACE_AT(3);
        }
        if (ep_tid == 0 && ep_traced)
            TPL_TRACE_PUT(100 + (a.epi == GT_QKV ? TR_QKV : a.epi == GT_GU ? TR_GU : a.trace_row_tag));
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (*s_fail && threadIdx.x == 0) {
        record_error(4u);
        for (int it = *s_consumed; it < *s_issued; ++it) mbar_wait(&full[it % NS], (unsigned)(it / NS) & 1u);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        TPL_TRACE_AT(3);
        TPL_TRACE_PUT(a.epi == GT_QKV ? TR_QKV : a.epi == GT_GU ? TR_GU : a.trace_row_tag);
    }
    if (warp == 1) {
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS));
    }
}

}  // namespace tpl
