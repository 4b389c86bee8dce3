// Internal declarations shared by the library's translation units.
#pragma once

#include <atomic>
#include <cstddef>
#include <cstdint>

#include "tpl.h"

#ifdef __CUDACC__
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#endif

namespace tpl {

constexpr int kGemvThreads = 512;          // 16 warps, one CTA per SM
constexpr int kGemvWarps = kGemvThreads / 32;
constexpr size_t kXSmemMax = 140 * 1024;   // activation slice staged per CTA
constexpr size_t kPartSmemMax = 64 * 1024; // per-round partial sums
constexpr int kAttnWarps = 4;              // warps per attention CTA (register-streamed kernel)
constexpr int kAttnStgWarps = 8;           // warps per CTA of the staged kernel
constexpr int kAttnTargetWarps = 1024;     // key-range splits across all (b, kv head) pairs
constexpr int kAttnMinKeys = 128;          // keys per split at least (when there are that many)
constexpr int kAttnMaxCtasPerPair = 64;
constexpr int kAttnSmsBound = 256;         // upper bound on SMs when sizing workspaces
constexpr int kTicketSlots = 10240;        // uint32 arrival counters at the workspace start
constexpr int kTicketAttn = 0;             // [0, 8192): attention pairs
constexpr int kTicketGemv = 8192;          // + 512 * op
constexpr int kMaxPairs = 8192;
constexpr int kMaxBatch = 64;              // decode tokens per call (tensor-core projections)
constexpr int kMaxBatchCuda = 16;          // with the mma.sync / FFMA projections (fp32 plans)

// Columns of the tensor-core decode projection's activation operand for B
// tokens: B hi rows and B lo rows when the activation is split, else B rows,
// rounded up to a valid MMA N (16, 32, 64, 128).
inline int gt_nx(int B, bool split) {
    const int rows = split ? 2 * B : B;
    return rows <= 16 ? 16 : rows <= 32 ? 32 : rows <= 64 ? 64 : 128;
}
// Floats per row of a cross-CTA piece of that projection (whole 16-token chunks).
inline int gt_stride(int B) { return 16 * ((B + 15) / 16); }
constexpr int kMaxRowBlocks = 512;
constexpr int kGemvTcMaxCtas = 256;        // CTAs of one tensor-core decode projection at most
constexpr int kGemvTcMaxTiles = 512;       // 128-row tiles per projection (one arrival counter each)

enum GemvOp { OP_QKV = 0, OP_O = 1, OP_GU = 2, OP_DOWN = 3 };

}  // namespace tpl

struct tpl_plan {
    tpl_dims d;
    int t;
    int nq_s, nkv_s, F_s, g, qkv_rows_s, esize;
    bool f32;
    int ld_h, ld_o, ld_f;                   // padded row lengths: hidden, n_q*d/t, ffn/t
    int64_t blk_qkv, blk_o, blk_gu, blk_d;  // byte stride between shard blocks
    int64_t off_qkv, off_o, off_gu, off_d, off_g1, off_g2, packed_bytes;
    std::atomic<long long> reductions;
    int gemv_mode;  // 0: mma.sync fragments (bf16); 1: fp32 FFMA; 2: bf16 FFMA; 3: tcgen05 + TMA (bf16);
                    // 4: per projection (default for bf16)
    int attn_prefill_mode;  // 0: tcgen05 (power-of-two group sizes); 1: mma.sync
    int prefill_split;      // TPL_SPLIT_* bits: prefill operands carried as bf16 hi + lo
    int prefill_tail;       // 1: a GEMM's partial last wave runs as half tiles
    int attn_decode_mode;   // 0: staged (g <= 8, pairs fit one wave); 1: register-streamed
    bool rope;
    double rope_theta[64];  // rope_base^(-2e/128), e < 64
};

namespace tpl {

// Geometry of one matrix-vector launch (rows split across CTAs, the K
// dimension split into segments (shards), split-K CTAs and K-groups of warps).
struct GemvGeom {
    int N;       // output rows
    int nseg;    // segments along K (t for row-parallel, 1 for column-parallel)
    int Kseg;    // columns per segment
    int nb;      // 128-column blocks per segment (last one ragged)
    int ksplit;  // CTAs along K per row block
    int wk, wr;  // warps: K-groups x row slots (wk * wr == 16)
    int rb;      // row blocks (grid = rb * ksplit)
    int ng;      // 8-row groups = ceil(N / 8)
    int cta_blocks;   // 128-column blocks of x staged per CTA (per segment span)
    int segs_per_cta; // whole segments per CTA (1 when a CTA holds part of one)
    int pieces;       // partial results per segment across split-K CTAs
    int rgc;          // row groups per warp per round
    int x_stride;     // bytes per token row of staged x
    size_t smem;      // dynamic shared memory bytes
    size_t gp_floats; // cross-CTA partial floats (0 when ksplit == 1)
};

// xparts: 1, or 2 when the activation is staged as bf16 hi + lo rows.
int gemv_geom(int N, int nseg, int Kseg, int B, int xbytes, int num_sms, GemvGeom *g, int xparts = 1);

struct AttnGeom {
    int pairs, nsplit, kps;  // pairs = B * n_kv; splits per pair; keys per split
    // the TMA-streamed kernel: blocks of kAttnTmaKeys keys per pair, CTAs of
    // the launch, CTAs per pair at most (sizes the partials)
    int nb = 0, grid = 0, cpp_max = 0;
};
constexpr int kAttnTmaKeys = 64;       // keys per block of the TMA-streamed decode attention
constexpr int kAttnTmaMaxCtas = 160;   // its CTAs per launch at most
// Geometry of the TMA-streamed kernel: grid = min(sms, kAttnTmaMaxCtas,
// pairs * nb) CTAs each taking an equal share of the pairs' blocks; a pair
// spans at most ceil(grid / pairs) + 1 CTAs.
void attn_geom_tma(int B, int nkv, int64_t keys, int sms, AttnGeom *a);
// keys: keys covered by the splits (S when the new token is added in the
// combine, S + 1 when it is read from the cache).
void attn_geom(int B, int nkv, int64_t keys, AttnGeom *a);
// Splits of the staged attention kernel: one CTA of kAttnStgWarps warps per
// SM, floor(sms / pairs) CTAs per pair (at least 64 keys per warp, at most
// kAttnMaxCtasPerPair).
void attn_geom_staged(int B, int nkv, int64_t keys, int sms, AttnGeom *a);

struct WsLayout {
    size_t tickets, q, o, h, act, ybuf0, ybuf1, P, knew, vnew, part_o, part_ml, gp;
    size_t xs;     // tcgen05 projections' operand x * gamma as bf16 hi rows, then lo rows [NX][hidden]
    size_t gpart;  // cross-CTA pieces of the tcgen05 projections
    size_t total;
};
int ws_layout(const tpl_plan *p, int B, int64_t S, WsLayout *w);

// Workspace of a prefill call over T tokens (byte offsets).
struct PrefillWs {
    size_t a_hi, a_lo;  // normalised activation, bf16 hi + lo [T][hidden] (reused for the MLP)
    size_t q;           // fp32 [T][n_q][d]
    size_t klo, vlo;    // bf16 rounding remainders of the new k/v [T][n_kv][d]
    size_t o, o_lo;     // attention output as bf16 hi + lo [T][n_q*d]
    size_t h;           // fp32 [T][hidden]
    size_t act;         // SwiGLU output, bf16 [T][ffn]
    size_t P;           // fp32 shard partials [t][T][hidden] (separate reduce mode)
    size_t total;
};
int prefill_ws_layout(const tpl_plan *p, int64_t T, PrefillWs *w);

int num_sms_current();  // multiprocessor count of the current device (cached)

}  // namespace tpl
