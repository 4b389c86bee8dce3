// Prefill projections on the 5th-generation tensor cores (tcgen05, TMEM).
//
// C[128-token tile][256-column tile] = A[tokens][K] . W[N][K]^T, bf16 in,
// fp32 accumulation in tensor memory.  Persistent: one CTA per SM walks a
// static list of output tiles.  320 threads:
//   warp 0     TMA producer (one thread): A and W tiles of 64 columns, 128-byte
//              swizzle, into an NS-stage shared-memory ring (no multicast;
//              every CTA loads its own tiles);
//   warp 1     allocates all 512 TMEM columns (two 256-column accumulators)
//              and issues tcgen05.mma (one thread): K-major shared-memory
//              descriptors, 4 MMAs of K = 16 per stage, a tcgen05.commit per
//              stage frees the stage, one per accumulation segment hands the
//              accumulator to the epilogue;
//   warps 2-9  epilogue: each reads its 32-lane quarter of TMEM (the lanes its
//              warp may access) for one 128-column half of the tile.
// An output tile is built from `nseg` accumulation segments.  Column-parallel
// projections have one.  The fused row-parallel projection ("Tensor parallel
// scaling curves", "What tensor parallelism actually splits") has one per
// shard (that shard's K slice): the epilogue keeps a running sum in
// registers, adding the shard partials in ascending shard order, so the result
// equals the separate partials summed by tpl_reduce_partials bit for bit.
// The two accumulators alternate, so the epilogue of one segment overlaps the
// MMAs of the next.  With SPLIT_A the activation comes as bf16 hi + lo tiles
// and each K step is two MMAs into the same accumulator.
//
// Every mbarrier wait is bounded; a wait that runs out records an error in
// the device error word, every role stops, copies already issued are waited
// for (bounded as well) and TMEM is released.
#pragma once

#include <cuda.h>

#include "tpl_common.cuh"
#include "tpl_internal.h"

namespace tpl {

constexpr int kGemmThreads = 320;
constexpr int kGemmEpiWarps = 8;
constexpr int kGemmMTile = 128;
constexpr int kGemmNTile = 256;
constexpr int kGemmHalfN = kGemmNTile / 2;  // the width of a half tile of the last wave
constexpr int kGemmKTile = 64;  // 128 bytes of bf16: one swizzle row
constexpr unsigned long long kWaitNs = 2000000000ull;  // 2 s: far above any healthy wait

enum { GEPI_F32 = 0, GEPI_QKV = 1, GEPI_GU = 2, GEPI_ROW = 3, GEPI_PARTIAL = 4 };

struct GemmArgs {
    CUtensorMap tm_a;   // A hi: [M][K] bf16 (2-D)
    CUtensorMap tm_a2;  // A lo (SPLIT_A)
    CUtensorMap tm_w;   // W: 2-D [N][K_pad] or 3-D [t][N][K_pad] (row-parallel)
    CUtensorMap tm_wh;  // the same weights in boxes of kGemmHalfN rows (half tiles)
    int M, N;           // output rows (tokens), output columns
    int k_blocks;       // 64-column blocks per accumulation segment
    int nseg;           // segments per output tile (t for the fused row split, else 1)
    int a_col_stride;   // A column offset between shards (row-parallel), in elements
    int w3d;            // weights are the 3-D per-shard map
    int m_tiles, n_tiles;
    int units;          // work units: full_units whole tiles, then two half tiles per remaining tile
    int full_units;     // tiles (m_tiles * n_tiles, * t in the separate row mode) done whole
    int epi;
    // epilogue outputs
    float *out32;       // GEPI_F32 / GEPI_ROW: [M][N]; GEPI_PARTIAL: [shards][M][N]
    void *out_act;      // GEPI_ROW: activation-type copy; GEPI_GU: act [M][N/2]
    int act_f32;
    const void *resid;  // GEPI_ROW
    int resid_f32;
    // QKV mapping: q fp32 [M][nq][hd]; k/v rounded to bf16 into the cache
    // (batch row 0, slot = pos0 + token) and their rounding remainders into
    // klo/vlo [M][nkv][hd] bf16
    float *q32;
    __nv_bfloat16 *klo, *vlo;
    __nv_bfloat16 *kc, *vc;
    int rps, nq, nq_s, nkv_s, hd, batch_cap;
    int64_t seq_cap;
    int64_t pos0;       // position of token row 0
    int rope;           // rotate q and k heads to their positions (hd = 128)
    double theta[64];   // rotary frequencies
};

__device__ __forceinline__ unsigned smem_u32(const void *p) { return (unsigned)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void mbar_init(uint64_t *bar, unsigned count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, unsigned bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}

__device__ __forceinline__ unsigned long long global_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Bounded wait for the phase of parity `parity`; false once kWaitNs have
// passed without it.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, unsigned parity) {
    const unsigned a = smem_u32(bar);
    unsigned long long t0 = 0;
    for (unsigned it = 0;; ++it) {
        unsigned done;
        asm volatile(
            "{ .reg .pred P; mbarrier.try_wait.parity.shared::cta.b64 P, [%1], %2; selp.u32 %0, 1, 0, P; }"
            : "=r"(done)
            : "r"(a), "r"(parity)
            : "memory");
        if (done) return true;
        if ((it & 255u) == 255u) {
            const unsigned long long now = global_ns();
            if (t0 == 0) t0 = now;
            else if (now - t0 > kWaitNs) return false;
        }
    }
}

__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *tm, int x, int y, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::
            "r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void tma_load_2d_hint(void *dst, const CUtensorMap *tm, int x, int y, uint64_t *bar,
                                                 uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1, {%2, "
        "%3}], [%4], %5;" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

__device__ __forceinline__ void tma_load_3d_hint(void *dst, const CUtensorMap *tm, int x, int y, int z, uint64_t *bar,
                                                 uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1, {%2, "
        "%3, %4}], [%5], %6;" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

__device__ __forceinline__ void tma_load_3d(void *dst, const CUtensorMap *tm, int x, int y, int z, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];" ::
            "r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
        : "memory");
}

// K-major, 128-byte-swizzle shared-memory matrix descriptor: rows of 128 B,
// 8-row groups 1024 B apart.
__device__ __forceinline__ uint64_t umma_desc(unsigned saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFF);
    d |= (uint64_t)1 << 16;            // leading byte offset (16 B; unused for swizzled K-major)
    d |= (uint64_t)(1024 >> 4) << 32;  // stride byte offset: 8 rows x 128 B
    d |= (uint64_t)1 << 46;            // descriptor version
    d |= (uint64_t)2 << 61;            // 128-byte swizzle
    return d;
}

// Instruction descriptor: bf16 x bf16 -> f32, both K-major, M x N.
__host__ __device__ constexpr uint32_t umma_idesc(int M, int N) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void umma(uint32_t tmem_d, uint64_t da, uint64_t db, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{ .reg .pred p; setp.ne.b32 p, %4, 0; tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p; }" ::"r"(tmem_d),
        "l"(da), "l"(db), "r"(idesc), "r"(acc));
}

__device__ __forceinline__ void umma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// 16 consecutive values of a row: activation-type or fp32 source.
__device__ __forceinline__ void load16(const void *p, int is_f32, int64_t i, float (&v)[16]) {
    if (is_f32) {
        const float4 *q = reinterpret_cast<const float4 *>(static_cast<const float *>(p) + i);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float4 f = q[k];
            v[4 * k] = f.x; v[4 * k + 1] = f.y; v[4 * k + 2] = f.z; v[4 * k + 3] = f.w;
        }
    } else {
        const uint4 *q = reinterpret_cast<const uint4 *>(static_cast<const __nv_bfloat16 *>(p) + i);
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            const uint4 u = q[k];
            const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                v[8 * k + 2 * e] = bf16lo(w[e]);
                v[8 * k + 2 * e + 1] = bf16hi(w[e]);
            }
        }
    }
}

__device__ __forceinline__ void store16_f32(float *dst, const float (&v)[16]) {
#pragma unroll
    for (int k = 0; k < 4; ++k)
        reinterpret_cast<float4 *>(dst)[k] = make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
}

__device__ __forceinline__ void store16_bf16(__nv_bfloat16 *dst, const float (&v)[16]) {
#pragma unroll
    for (int k = 0; k < 2; ++k)
        reinterpret_cast<uint4 *>(dst)[k] =
            make_uint4(pack_bf16x2(v[8 * k], v[8 * k + 1]), pack_bf16x2(v[8 * k + 2], v[8 * k + 3]),
                       pack_bf16x2(v[8 * k + 4], v[8 * k + 5]), pack_bf16x2(v[8 * k + 6], v[8 * k + 7]));
}

template <bool SPLIT_A>
struct GemmSmem {
    static constexpr int A_BYTES = kGemmMTile * kGemmKTile * 2;  // 16 KB
    static constexpr int W_BYTES = kGemmNTile * kGemmKTile * 2;  // 32 KB
    static constexpr int STAGE = A_BYTES * (SPLIT_A ? 2 : 1) + W_BYTES;
    static constexpr int NS = (200 * 1024) / STAGE;
    static constexpr int BYTES = NS * STAGE + 1024 /* alignment */ + 256 /* barriers */;
};

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Unit u -> tile origin, the shard of a separate-mode unit, and which half
// of the tile's columns a half unit covers (-1: the whole tile).  Tiles past
// full_units are done as two units of kGemmHalfN columns each, so that the
// last, partial wave of tiles spreads over twice as many SMs.
__device__ __forceinline__ void gemm_unit(const GemmArgs &a, int u, int &m0, int &n0, int &shard, int &half) {
    half = -1;
    if (u >= a.full_units) {
        const int h = u - a.full_units;
        u = a.full_units + (h >> 1);
        half = h & 1;
    }
    const int mt = u % a.m_tiles;
    const int r = u / a.m_tiles;
    m0 = mt * kGemmMTile;
    n0 = (r % a.n_tiles) * kGemmNTile;
    shard = r / a.n_tiles;
}

// Epilogue of one 16-column chunk of a single-segment tile.
__device__ __forceinline__ void gemm_epi_chunk(const GemmArgs &a, const float (&v)[16], int row, int col, int shard) {
    if (row >= a.M || col >= a.N) return;
    const bool full16 = col + 16 <= a.N;  // ragged last chunk: scalar stores
    if (a.epi == GEPI_PARTIAL || a.epi == GEPI_F32) {
        float *dst = a.out32 + ((int64_t)(a.epi == GEPI_PARTIAL ? shard : 0) * a.M + row) * a.N + col;
        if (full16) store16_f32(dst, v);
        else
#pragma unroll
            for (int i = 0; i < 16; ++i)
                if (col + i < a.N) dst[i] = v[i];
    } else if (a.epi == GEPI_GU) {
        // rows interleave gate and up: (g, u) pairs -> silu(g) * u
        const int64_t base = (int64_t)row * (a.N / 2) + col / 2;
        if (full16 && !a.act_f32) {
            const uint4 u = make_uint4(pack_bf16x2(silu(v[0]) * v[1], silu(v[2]) * v[3]),
                                       pack_bf16x2(silu(v[4]) * v[5], silu(v[6]) * v[7]),
                                       pack_bf16x2(silu(v[8]) * v[9], silu(v[10]) * v[11]),
                                       pack_bf16x2(silu(v[12]) * v[13], silu(v[14]) * v[15]));
            *reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(a.out_act) + base) = u;
        } else {
#pragma unroll
            for (int i = 0; i < 16; i += 2)
                if (col + i + 1 < a.N) store_act(a.out_act, a.act_f32, base + i / 2, silu(v[i]) * v[i + 1]);
        }
    } else if (a.epi == GEPI_QKV) {  // a 16-column chunk never straddles a head
        const int s = col / a.rps, l = col % a.rps;
        const int qd = a.nq_s * a.hd, kd = a.nkv_s * a.hd;
        if (l < qd) {
            const int head = s * a.nq_s + l / a.hd, dim = l % a.hd;
            store16_f32(a.q32 + ((int64_t)row * a.nq + head) * a.hd + dim, v);
        } else {
            const bool isk = l < qd + kd;
            const int ll = isk ? l - qd : l - qd - kd;
            const int kvl = ll / a.hd, dim = ll % a.hd;
            const int nkv = a.nkv_s * (a.nq / a.nq_s);
            float hi[16], lo[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                hi[i] = __bfloat162float(__float2bfloat16_rn(v[i]));
                lo[i] = v[i] - hi[i];
            }
            __nv_bfloat16 *cc = isk ? a.kc : a.vc;
            store16_bf16(cc + (((int64_t)s * a.batch_cap) * a.nkv_s + kvl) * a.seq_cap * a.hd +
                             (a.pos0 + row) * a.hd + dim,
                         hi);
            __nv_bfloat16 *fl = isk ? a.klo : a.vlo;
            store16_bf16(fl + ((int64_t)row * nkv + s * a.nkv_s + kvl) * a.hd + dim, lo);
        }
    }
}

// Final store of a summed row-split chunk: out = resid + sum.
__device__ __forceinline__ void gemm_row_store(const GemmArgs &a, float (&v)[16], int row, int col) {
    if (row >= a.M || col >= a.N) return;
    const int64_t base = (int64_t)row * a.N + col;
    if (col + 16 <= a.N) {
        if (a.resid) {
            float r[16];
            load16(a.resid, a.resid_f32, base, r);
#pragma unroll
            for (int i = 0; i < 16; ++i) v[i] = r[i] + v[i];
        }
        if (a.out32) store16_f32(a.out32 + base, v);
        if (a.out_act) {
            if (a.act_f32) store16_f32(static_cast<float *>(a.out_act) + base, v);
            else store16_bf16(static_cast<__nv_bfloat16 *>(a.out_act) + base, v);
        }
    } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            if (col + i >= a.N) continue;
            float o = v[i];
            if (a.resid) o = load_act(a.resid, a.resid_f32, base + i) + o;
            if (a.out32) a.out32[base + i] = o;
            if (a.out_act) store_act(a.out_act, a.act_f32, base + i, o);
        }
    }
}

template <bool SPLIT_A, bool ROWSUM>
__global__ void __launch_bounds__(kGemmThreads, 1) gemm_tc_kernel(const __grid_constant__ GemmArgs a) {
    using SM = GemmSmem<SPLIT_A>;
    constexpr int NS = SM::NS;
    constexpr int TMEM_COLS = 2 * kGemmNTile;
    extern __shared__ __align__(1024) unsigned char gsm_raw[];
    unsigned char *gsm = reinterpret_cast<unsigned char *>(((uintptr_t)gsm_raw + 1023) & ~(uintptr_t)1023);
    uint64_t *full = reinterpret_cast<uint64_t *>(gsm + NS * SM::STAGE);
    uint64_t *empty = full + NS;
    uint64_t *acc_full = empty + NS;  // [2]
    uint64_t *acc_empty = acc_full + 2;  // [2]
    uint64_t *fin = acc_empty + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(fin + 1);
    volatile int *s_fail = reinterpret_cast<volatile int *>(tmem_slot + 1);
    int *s_issued = const_cast<int *>(s_fail) + 1;    // stages the producer filled
    int *s_consumed = const_cast<int *>(s_fail) + 2;  // stages the MMA issuer took

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], kGemmEpiWarps);
        }
        mbar_init(fin, 1);
        *s_fail = 0;
        *s_issued = 0;
        *s_consumed = 0;
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

    pdl_wait();
    pdl_trigger();

    if (warp == 0) {
        if (lane == 0) {
            constexpr unsigned TX = SM::A_BYTES * (SPLIT_A ? 2 : 1) + SM::W_BYTES;
            constexpr unsigned TX_HALF = TX - SM::W_BYTES / 2;
            int it = 0;
            for (int u = blockIdx.x; u < a.units && !*s_fail; u += gridDim.x) {
                int m0, n0, su, half;
                gemm_unit(a, u, m0, n0, su, half);
                const CUtensorMap *wm = half < 0 ? &a.tm_w : &a.tm_wh;
                const int wn = half < 0 ? n0 : n0 + half * kGemmHalfN;
                for (int seg = 0; seg < a.nseg && !*s_fail; ++seg) {
                    const int sh = su + seg;
                    for (int kb = 0; kb < a.k_blocks; ++kb, ++it) {
                        const int s = it % NS;
                        const unsigned ph = (unsigned)(it / NS) & 1u;
                        if (*s_fail || !mbar_wait(&empty[s], ph ^ 1u)) {
                            *s_fail = 1;
                            break;
                        }
                        unsigned char *st = gsm + s * SM::STAGE;
                        mbar_expect_tx(&full[s], half < 0 ? TX : TX_HALF);
                        const int ax = sh * a.a_col_stride + kb * kGemmKTile;
                        tma_load_2d(st, &a.tm_a, ax, m0, &full[s]);
                        if (SPLIT_A) tma_load_2d(st + SM::A_BYTES, &a.tm_a2, ax, m0, &full[s]);
                        unsigned char *wdst = st + SM::A_BYTES * (SPLIT_A ? 2 : 1);
                        if (a.w3d) tma_load_3d(wdst, wm, kb * kGemmKTile, wn, sh, &full[s]);
                        else tma_load_2d(wdst, wm, kb * kGemmKTile, wn, &full[s]);
                    }
                }
            }
            *s_issued = it;
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t IDESC_FULL = umma_idesc(kGemmMTile, kGemmNTile);
            constexpr uint32_t IDESC_HALF = umma_idesc(kGemmMTile, kGemmHalfN);
            int it = 0, c = 0;
            for (int u = blockIdx.x; u < a.units && !*s_fail; u += gridDim.x) {
                // a half unit is an N = 128 product into the accumulator's
                // first 128 columns, over the same K steps in the same order
                const uint32_t IDESC = u < a.full_units ? IDESC_FULL : IDESC_HALF;
                for (int seg = 0; seg < a.nseg && !*s_fail; ++seg, ++c) {
                    const int b = c & 1;
                    const unsigned use = (unsigned)(c >> 1);
                    if (*s_fail || !mbar_wait(&acc_empty[b], (use & 1u) ^ 1u)) {
                        *s_fail = 1;
                        break;
                    }
                    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                    const uint32_t dcol = tmem + (uint32_t)(b * kGemmNTile);
                    bool ok = true;
                    for (int kb = 0; kb < a.k_blocks; ++kb, ++it) {
                        const int s = it % NS;
                        const unsigned ph = (unsigned)(it / NS) & 1u;
                        if (*s_fail || !mbar_wait(&full[s], ph)) {
                            *s_fail = 1;
                            ok = false;
                            break;
                        }
                        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                        const unsigned sa = smem_u32(gsm + s * SM::STAGE);
                        const unsigned sw = sa + SM::A_BYTES * (SPLIT_A ? 2 : 1);
#pragma unroll
                        for (int k = 0; k < kGemmKTile / 16; ++k) {
                            const uint64_t db = umma_desc(sw + 32 * k);
                            umma(dcol, umma_desc(sa + 32 * k), db, IDESC, (kb > 0 || k > 0) ? 1u : 0u);
                            if (SPLIT_A) umma(dcol, umma_desc(sa + SM::A_BYTES + 32 * k), db, IDESC, 1u);
                        }
                        umma_commit(&empty[s]);  // stage free once these MMAs complete
                    }
                    if (!ok) break;
                    umma_commit(&acc_full[b]);  // accumulator b holds this segment
                }
            }
            *s_consumed = it;
            // every MMA this thread issued has completed once `fin` flips
            umma_commit(fin);
            if (!mbar_wait(fin, 0)) *s_fail = 1;
        }
    } else {
        // ---- epilogue: warp w reads TMEM lanes 32*(w % 4).. (its accessible
        // quarter) for columns [128*h, 128*h + 128) of the tile ----
        const int q = warp & 3, hf = (warp - 2) >> 2;
        const uint32_t lane_base = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(hf * 128);
        int c = 0;
        for (int u = blockIdx.x; u < a.units && !*s_fail; u += gridDim.x) {
            int m0, n0, su, half;
            gemm_unit(a, u, m0, n0, su, half);
            const int row = m0 + 32 * q + lane;
            // a half unit's columns sit in accumulator columns [0, 128): the
            // warps of the first column half store them, the others (cb = N)
            // only keep the accumulator hand-off in step; so do warps whose
            // columns all lie past N
            const int cb = half < 0 ? n0 + hf * 128 : (hf == 0 ? n0 + half * kGemmHalfN : a.N);
            const bool idle = cb >= a.N;
            float sum[ROWSUM ? 128 : 1];  // running sum of the shard partials (fused row split)
            bool ok = true;
            for (int seg = 0; seg < a.nseg; ++seg, ++c) {
                const int b = c & 1;
                const unsigned use = (unsigned)(c >> 1);
                if (*s_fail || !mbar_wait(&acc_full[b], use & 1u)) {
                    *s_fail = 1;
                    ok = false;
                    break;
                }
                asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                const uint32_t taddr = lane_base + (uint32_t)(b * kGemmNTile);
                if (idle) {
                    // nothing of this unit in the second column half
                } else if constexpr (ROWSUM) {
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        float v[16];
                        tmem_ld16(taddr + 16 * j, v);
#pragma unroll
                        // -0 is the additive identity (x + -0 == x for every x,
                        // +-0 included): segment 0 stores its partial unchanged
                        for (int i = 0; i < 16; ++i) sum[16 * j + i] = (seg == 0 ? -0.f : sum[16 * j + i]) + v[i];
                    }
                } else if (a.rope && a.epi == GEPI_QKV && (cb % a.rps) < (a.nq_s + a.nkv_s) * a.hd) {
                    // this warp's 128 columns are one q or k head: turn each
                    // pair (e, e + 64) by the row's rotary angle
                    const double pos = (double)(a.pos0 + row);
                    for (int j = 0; j < 4; ++j) {
                        float v0[16], v1[16];
                        tmem_ld16(taddr + 16 * j, v0);
                        tmem_ld16(taddr + 16 * (j + 4), v1);
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            float cs, sn;
                            rope_cs(pos, a.theta[16 * j + i], cs, sn);
                            const float x0 = v0[i], x1 = v1[i];
                            v0[i] = x0 * cs - x1 * sn;
                            v1[i] = x1 * cs + x0 * sn;
                        }
                        gemm_epi_chunk(a, v0, row, cb + 16 * j, su);
                        gemm_epi_chunk(a, v1, row, cb + 64 + 16 * j, su);
                    }
                } else {
                    for (int j = 0; j < 8; ++j) {
                        float v[16];
                        tmem_ld16(taddr + 16 * j, v);
                        gemm_epi_chunk(a, v, row, cb + 16 * j, su);
                    }
                }
                asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
                __syncwarp();
                if (lane == 0) mbar_arrive(&acc_empty[b]);
            }
            if (!ok) break;
            if constexpr (ROWSUM) {
                if (idle) continue;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    float v[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) v[i] = sum[16 * j + i];
                    gemm_row_store(a, v, row, cb + 16 * j);
                }
            }
        }
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (*s_fail && threadIdx.x == 0) {
        record_error(4u);
        // let copies that were issued but never consumed land before the
        // shared memory goes away (bounded as well)
        for (int it = *s_consumed; it < *s_issued; ++it) mbar_wait(&full[it % NS], (unsigned)(it / NS) & 1u);
    }
    __syncthreads();
    if (warp == 1) {
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS));
    }
}

}  // namespace tpl
