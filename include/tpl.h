/*
 * tpl -- a single-device Megatron-style tensor-parallel transformer layer.
 *
 * The problem, as the pages state it: an input x, a shard degree t and the
 * layer dimensions go in; the output equals that of the unsharded layer.
 * Inside, the layer is computed the tensor-parallel way:
 *   - Q/K/V and gate/up projections are split by output columns into t
 *     shards, Q/K/V by whole attention heads ("Tensor parallel scaling
 *     curves", section "What tensor parallelism actually splits"; shard s
 *     owns the contiguous query heads [s*n_q/t, (s+1)*n_q/t));
 *   - each shard attends over its own heads only, with no exchange (same
 *     section);
 *   - the O and down projections are split by input rows, so each shard
 *     yields a full-size partial sum, and the t partials are added -- the
 *     arithmetic of the all-reduce, two per layer, 2L per forward pass (same
 *     section; "Tensor Parallelism Fundamentals", section "Mechanics of
 *     Matrix Slicing").
 * All t shards live in one device's memory: a shard is a weight and KV-cache
 * layout, and the partial-sum reduction runs on the device, fused into the
 * epilogue of the row-parallel kernels (TPL_REDUCE_FUSED) or as a separate
 * ordered reduction (TPL_REDUCE_SEPARATE, kept for comparison).  The two
 * modes produce bitwise identical results.
 *
 * Conventions for every call:
 *   - Device pointers are plain CUDA device addresses; host pointers are
 *     marked "host".  The caller owns every buffer (weights, packed weights,
 *     KV caches, activations, workspace); the library never allocates device
 *     memory and owns only the host-side plan.
 *   - `stream` is a cudaStream_t passed as void*.  Calls only enqueue work on
 *     it and return; nothing synchronises except tpl_last_device_error.
 *   - Calls return a status (TPL_OK or a TPL_E* code).  Arguments are
 *     validated on the host before anything is launched; on an error nothing
 *     is launched.  No C++ exception crosses this interface.
 *   - Activations use the "activation type": bf16 by default, fp32 when the
 *     plan's flags contain TPL_FP32_WEIGHTS.  The KV cache is always bf16.
 *   - Weights use the nn.Linear orientation W[out][in], row-major.
 */
#ifndef TPL_H
#define TPL_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif
#if defined(__GNUC__)
#pragma GCC visibility push(default)
#endif

/* ---- status codes ------------------------------------------------------ */
#define TPL_OK 0
#define TPL_EINVAL 1        /* null pointer, negative size, bad enum value      */
#define TPL_EINDIVISIBLE 2  /* t not in {1,2,4,8}, or t does not divide n_q_heads,
                               n_kv_heads or ffn                                 */
#define TPL_EWORKSPACE 3    /* workspace smaller than tpl_workspace_size()       */
#define TPL_ENOMEM 4        /* a caller-provided capacity is too small (packed
                               buffer, KV capacity)                              */
#define TPL_ECUDA 5         /* a CUDA call or kernel launch failed               */
#define TPL_EDEVICE 6       /* a kernel reported an inconsistency (device error
                               word, read by tpl_last_device_error)              */
#define TPL_EUNSUPPORTED 7  /* valid dimensions this build does not implement
                               (head_dim != 128, group size > 16, dims not a
                               multiple of 8; more than 64 decode tokens per
                               call, more than 16 with fp32 weights)             */
#define TPL_ENOFIT 8        /* tpl_auto_t: no admissible degree fits the budget  */

/* ---- flags ------------------------------------------------------------- */
#define TPL_NORM 1u          /* pre-RMSNorm before QKV and before gate/up       */
#define TPL_RESIDUAL 2u      /* residual adds after O and after down            */
#define TPL_FP32_WEIGHTS 4u  /* fp32 weights and activations (KV stays bf16)    */
#define TPL_ROPE 8u          /* rotary position embedding of q and k (below)    */

#define TPL_REDUCE_FUSED 0    /* t-way sum inside the row-parallel epilogue     */
#define TPL_REDUCE_SEPARATE 1 /* partials to memory, then tpl_reduce_partials   */

typedef void *tpl_stream; /* a cudaStream_t */

/* Layer dimensions.  head_dim must be 128; hidden and ffn/t multiples of 8.
 * With TPL_ROPE, q and the new k of every token are turned to the token's
 * position before attention and before k enters the cache: for e < 64 the
 * pair (v[e], v[e + 64]) is rotated by the angle pos * rope_base^(-2e/128)
 * (the rotary embedding of RoFormer, Su et al. 2021, in the half-split
 * pairing of the Llama family; the pages do not name a position encoding, so
 * it is off unless flagged).  rope_base must be > 1 when TPL_ROPE is set and
 * is ignored otherwise. */
typedef struct {
    int32_t hidden, n_q_heads, n_kv_heads, head_dim, ffn, n_layers;
    float rms_eps;
    uint32_t flags; /* TPL_NORM | TPL_RESIDUAL | TPL_FP32_WEIGHTS | TPL_ROPE */
    float rope_base;
} tpl_dims;

typedef struct tpl_plan tpl_plan; /* opaque, host-owned by the library */

/* Footprints of a plan.  All sizes are per layer unless stated. */
typedef struct {
    int32_t t;
    int32_t q_heads_per_shard, kv_heads_per_shard, ffn_per_shard, group_size;
    int32_t qkv_rows_per_shard;        /* (n_q/t + 2 n_kv/t) * head_dim          */
    int32_t elem_bytes;                /* weight/activation element size: 2 or 4 */
    int64_t layer_params_per_shard;    /* Wq,Wk,Wv rows + Wo cols + Wg,Wu rows + Wd cols */
    int64_t layer_weight_bytes_per_shard;
    int64_t packed_layer_bytes;        /* bytes tpl_pack_layer writes (all shards + gains) */
    int64_t reductions_per_step;       /* 2 * n_layers                             */
} tpl_plan_info;

/* Unsharded weights of one layer on the device, nn.Linear orientation, in the
 * activation type: wq [n_q*d][H], wk/wv [n_kv*d][H], wo [H][n_q*d],
 * wg/wu [F][H], wd [H][F].  gamma_* are fp32 [H]; NULL means all ones.
 * For an MLP-only plan (n_q_heads used only for sizing) wq..wo may be NULL. */
typedef struct {
    const void *wq, *wk, *wv, *wo, *wg, *wu, *wd;
    const float *gamma_attn, *gamma_mlp;
} tpl_layer_weights;

/* The KV cache of one layer, all shards, bf16, shard-major:
 *   k, v: [t][batch_cap][n_kv/t][seq_cap][head_dim]
 * (shard s's part is a contiguous block, as it would be on its own GPU; the
 * per-GPU size is the formula of "Tensor Parallelism Fundamentals", section
 * "Memory Overhead and Communication Bottlenecks"). */
typedef struct {
    void *k, *v;
    int32_t batch_cap;
    int64_t seq_cap;
} tpl_kv;

/* ---- planning (host only; no GPU needed) -------------------------------- */

/* Create a plan for dims `*dims` and degree t.  Validates the shard maps of
 * "Tensor parallel scaling curves" ("What tensor parallelism actually
 * splits"): t in {1,2,4,8} ("Tensor Parallelism" docs: the size is 1, 2, 4 or
 * 8), t | n_q_heads, t | n_kv_heads, t | ffn, n_kv_heads | n_q_heads.
 * *out receives a plan to be released with tpl_plan_destroy. */
int tpl_plan_create(const tpl_dims *dims, int32_t t, tpl_plan **out);
void tpl_plan_destroy(tpl_plan *plan);

/* Plan options (host).  TPL_OPT_GEMV_MODE selects the kernels of the bf16
 * decode projections: 0 = register-streamed weights on mma.sync, 2 = FFMA on
 * the CUDA cores (kept to measure against), 3 = weights streamed by TMA into
 * a shared-memory ring and multiplied on the 5th-generation tensor cores
 * (tcgen05, accumulators in TMEM; their operand is x * gamma as bf16 hi + lo,
 * written by the preceding row-parallel kernel inside a layer or by a small
 * kernel, and the RMSNorm factor 1/rms is applied to their results), 4 = the
 * default: the tcgen05 kernels for every projection at any token count on
 * layers with at least 1 GiB of weights and from 7 tokens on any layer,
 * mma.sync otherwise (the choice that measured faster on B200; layers mixing
 * the two families measured slower than either).  Above 16 tokens every mode runs
 * the tcgen05 kernels.  fp32 plans always use FFMA.  TPL_OPT_PREFILL_ATTN selects the prefill attention kernel:
 * 0 = 5th-generation tensor cores (tcgen05, TMEM; the default when the
 * query group size is a power of two), 1 = mma.sync (any group size; kept to
 * measure against).  TPL_OPT_DECODE_ATTN selects the decode attention kernel:
 * 0 = keys staged through a per-warp shared-memory ring (the default for
 * query groups of at most 8 heads when every (shard, sequence, kv head) pair
 * gets at least two CTAs in one wave of SMs, and the cache streamed by TMA
 * (below) when the pairs fit one wave and each has at least 8192 cached keys;
 * other shapes use the register kernel), 1 = keys streamed into registers
 * (any shape), 2 = the cache
 * streamed by TMA into a shared-memory ring, every SM taking an equal share
 * of all pairs' 64-key blocks (groups of at most 8 heads and S >= 1; other
 * cases as 0).
 * TPL_OPT_PREFILL_SPLIT chooses, per prefill projection, whether its
 * activation operand is carried as two bf16 parts (hi + lo, about 16
 * mantissa bits, two products per tile) or one (rounded to bf16, one
 * product): a bit mask of TPL_SPLIT_QKV (the normalised x into QKV),
 * TPL_SPLIT_O (the attention output into O) and TPL_SPLIT_GU (the normalised
 * h into gate/up); the down projection's operand (act) is always one part.
 * Default TPL_SPLIT_DEFAULT.
 * TPL_OPT_PREFILL_TAIL: 1 (the default) runs a prefill projection's last,
 * partial wave of 128 x 256 output tiles as 128 x 128 half tiles when it
 * fills at most half the SMs (two units per tile over the same K steps in
 * the same order: the results are bit-identical to whole tiles); 0 keeps
 * every tile whole (kept to measure against and to check that identity).
 * Returns TPL_EINVAL for an unknown option or value. */
#define TPL_OPT_GEMV_MODE 1
#define TPL_OPT_PREFILL_ATTN 2
#define TPL_OPT_DECODE_ATTN 3
#define TPL_OPT_PREFILL_SPLIT 4
#define TPL_OPT_PREFILL_TAIL 5
#define TPL_SPLIT_QKV 1
#define TPL_SPLIT_O 2
#define TPL_SPLIT_GU 4
#define TPL_SPLIT_DEFAULT (TPL_SPLIT_QKV | TPL_SPLIT_O | TPL_SPLIT_GU)
int tpl_plan_set_option(tpl_plan *plan, int32_t option, int32_t value);

/* Footprints (host) -- see tpl_plan_info. */
int tpl_plan_info_get(const tpl_plan *plan, tpl_plan_info *out);

/* Shard maps (host arrays, each may be NULL):
 *   q_shard[n_q], q_local[n_q]: shard and local index of query head h;
 *   kv_shard[n_kv]: shard of kv head j;
 *   ffn_shard[ffn]: shard of ffn column c;
 *   packed_offsets[4*t + 2]: byte offsets inside a packed layer of the blocks
 *     Wqkv[s], Wo[s], Wgu[s], Wd[s] (s = 0..t-1, in that order) followed by
 *     gamma_attn and gamma_mlp. */
int tpl_plan_maps(const tpl_plan *plan, int32_t *q_shard, int32_t *q_local, int32_t *kv_shard,
                  int32_t *ffn_shard, int64_t *packed_offsets);

/* Per-GPU KV bytes of the whole model: 2*n_layers*n_kv*head_dim*seq*
 * bytes_per_elem*batch / t ("Tensor Parallelism Fundamentals", "Memory
 * Overhead and Communication Bottlenecks").  Returns -1 on invalid input or
 * when t does not divide the total. */
int64_t tpl_kv_bytes(const tpl_dims *dims, int32_t t, int64_t batch, int64_t seq,
                     int32_t bytes_per_elem);

/* Per-GPU bytes at degree t of the n_layers layers' weights (each shard's
 * slices, bytes_per_elem per parameter) plus the KV cache of tpl_kv_bytes:
 * the two footprints "Tensor Parallelism Fundamentals" (section "Memory
 * Overhead and Communication Bottlenecks") divides by t.  Embeddings and
 * activations are not counted.  Host only.  -1 on invalid input or when t
 * does not divide n_q_heads, n_kv_heads and ffn. */
int64_t tpl_footprint_bytes(const tpl_dims *dims, int32_t t, int64_t batch, int64_t seq,
                            int32_t bytes_per_elem);

/* The "Auto" rule of the "Tensor Parallelism" docs (section "Auto"): the
 * smallest power of two t in {1, 2, 4, 8}, t <= max_t (the GPUs one model may
 * use), that divides n_q_heads, n_kv_heads and ffn and whose
 * tpl_footprint_bytes fits "comfortably": footprint <= budget_bytes *
 * (1 - headroom), headroom in [0, 1) chosen by the caller.  With budget_bytes
 * <= 0 (the target's memory cannot be seen) it is the largest such t, as the
 * docs' remote-node fallback.  *t_out (host) receives t; TPL_ENOFIT (and
 * *t_out = 0) when no admissible t fits, TPL_EINVAL on invalid input. */
int tpl_auto_t(const tpl_dims *dims, int64_t budget_bytes, double headroom, int64_t batch, int64_t seq,
               int32_t bytes_per_elem, int32_t max_t, int32_t *t_out);

/* The per-token time model of "Tensor parallel scaling curves", section "The
 * scaling math": T(N) = T_compute/N + T_memory/N + 2L * T_allreduce(N), with
 * T_allreduce(N) = latency + 2 (N-1)/N * message_bytes / link_bytes_per_s
 * (a ring all-reduce moves about 2 (N-1)/N of the message per GPU, section
 * "What tensor parallelism actually splits") and no all-reduce at N = 1.
 * All times in seconds. */
typedef struct {
    double t_compute, t_memory; /* the single-GPU terms, as given            */
    double t_allreduce;         /* one call at N                              */
    double t_comm;              /* 2L * t_allreduce                           */
    double t_total;             /* T(N)                                       */
    double speedup;             /* T(1) / T(N)                                */
    double comm_share;          /* t_comm / t_total                           */
} tpl_tp_estimate;
int tpl_tp_estimate_get(double t_compute, double t_memory, int32_t n, int32_t layers, double message_bytes,
                        double latency_s, double link_bytes_per_s, tpl_tp_estimate *out);

/* The single-GPU terms of one decode step of the whole model (dims->n_layers
 * layers, batch sequences each attending over seq cached tokens), for
 * tpl_tp_estimate_get: t_compute = 2 * params * batch / flops_per_s (one
 * multiply-add per weight per token), t_memory = tpl_footprint_bytes(t = 1) /
 * hbm_bytes_per_s (every weight and the cache read once).  Host outputs. */
int tpl_decode_times(const tpl_dims *dims, int64_t batch, int64_t seq, int32_t bytes_per_elem,
                     double flops_per_s, double hbm_bytes_per_s, double *t_compute, double *t_memory);

/* Bytes of one layer's K (or V) buffer for tpl_kv with the given capacities. */
int64_t tpl_kv_layer_bytes(const tpl_plan *plan, int32_t batch_cap, int64_t seq_cap);

/* Workspace bytes needed by the decode calls for batch B and cached length S
 * (both reduce modes). */
int tpl_workspace_size(const tpl_plan *plan, int32_t batch, int64_t seq, size_t *out);

/* Workspace bytes needed by tpl_prefill_layer for a chunk of T tokens (both
 * reduce modes; the separate mode's t partial sums [t][T][hidden] fp32 are
 * the largest part).  TPL_EINVAL for T <= 0. */
int tpl_prefill_workspace_size(const tpl_plan *plan, int32_t T, size_t *out);

/* Byte offsets, inside a prefill workspace for T tokens, of the
 * intermediates the last tpl_prefill_layer call on it left behind:
 *   offsets[0]  q     fp32 [T][n_q][d]
 *   offsets[1]  o     attention output, bf16 high part [T][n_q*d]
 *   offsets[2]  h     fp32 [T][hidden] (after the first reduction)
 *   offsets[3]  act   SwiGLU output, bf16 [T][ffn]
 *   offsets[4]  o_lo  attention output, bf16 remainder: o = o + o_lo
 * (for inspection and tests; the pages define these as the layer's
 * intermediate values).  offsets: host array of 5. */
int tpl_prefill_intermediates(const tpl_plan *plan, int32_t T, size_t *offsets);

/* ---- device calls ------------------------------------------------------- */

/* Zero the workspace's bookkeeping words (cross-block arrival counters).
 * Call once after allocating a workspace (or zero the whole buffer); kernels
 * leave the counters at zero afterwards. */
int tpl_workspace_init(const tpl_plan *plan, void *ws, size_t ws_bytes, tpl_stream stream);

/* Rearrange one layer's unsharded weights into the plan's packed shard
 * layout (`packed`, packed_bytes >= info.packed_layer_bytes), every row
 * zero-padded to a whole number of 128-column blocks:
 *   Wqkv[s] = rows [q heads of s | k heads of s | v heads of s] of Wq/Wk/Wv
 *   Wo[s]   = Wo[:, s*(n_q/t)*d : (s+1)*(n_q/t)*d]           (row split)
 *   Wgu[s]  = rows Wg[c], Wu[c] interleaved for c in shard s's ffn columns
 *   Wd[s]   = Wd[:, s*F/t : (s+1)*F/t]                        (row split)
 * then gamma_attn, gamma_mlp (fp32).  "Tensor parallel scaling curves",
 * "What tensor parallelism actually splits". */
int tpl_pack_layer(const tpl_plan *plan, const tpl_layer_weights *w, void *packed,
                   size_t packed_bytes, tpl_stream stream);

/* Copy an unsharded cache [batch_cap][n_kv][seq_cap][d] (bf16) into the
 * shard-major layout of tpl_kv (both device buffers, same byte size). */
int tpl_pack_kv(const tpl_plan *plan, const void *unsharded, void *sharded, int32_t batch_cap,
                int64_t seq_cap, tpl_stream stream);

/* One decode step of one layer for B sequences with S cached tokens each
 * (the new token is position S; requires S < kv->seq_cap, B <= batch_cap;
 * B <= 64, and B <= 16 for fp32 plans.  Above 16 tokens the projections run
 * on the tensor-core kernel whatever TPL_OPT_GEMV_MODE says):
 *   a = RMSNorm(x)            [TPL_NORM]
 *   q|k|v = column-parallel projection of a, k/v written to slot S
 *   o = owned-head GQA attention over the S+1 positions
 *   h = x + sum_s o_s Wo[s]^T  (reduction point 1)   [+x if TPL_RESIDUAL]
 *   m = RMSNorm(h)            [TPL_NORM]
 *   y = h + sum_s (silu(m Wg_s^T) * (m Wu_s^T)) Wd[s]^T (reduction point 2)
 * x, y: [B][hidden] activation type; y32: fp32 [B][hidden] or NULL.
 * reduce_mode: TPL_REDUCE_FUSED or TPL_REDUCE_SEPARATE. */
int tpl_decode_layer(tpl_plan *plan, const void *packed, const tpl_kv *kv, const void *x,
                     int32_t B, int64_t S, void *y, float *y32, void *ws, size_t ws_bytes,
                     int32_t reduce_mode, tpl_stream stream);

/* n_layers decode steps: layer l reads layer l-1's output.  packed_per_layer
 * and kv_per_layer are host arrays of n_layers entries.  Adds 2 * n_layers to
 * the plan's reduction counter ("Tensor parallel scaling curves": 2L
 * all-reduce points per forward pass). */
int tpl_decode_stack(tpl_plan *plan, const void *const *packed_per_layer, const tpl_kv *kv_per_layer,
                     const void *x, int32_t B, int64_t S, void *y, float *y32, void *ws,
                     size_t ws_bytes, int32_t reduce_mode, tpl_stream stream);

/* Prefill of one layer over T tokens of one sequence starting at position 0
 * (causal inside the chunk: token i sees positions 0..i), writing K/V cache
 * slots 0..T-1 of batch row 0 ("Tensor parallel scaling curves", sections
 * "What tensor parallelism actually splits" and "Prefill vs decode:
 * different curves": the same splits as decode, over many tokens, so every
 * projection is a matrix product):
 *   a = RMSNorm(x); q|k|v = a Wqkv[s]^T per shard; causal attention on owned
 *   heads; h = x + sum_s o_s Wo[s]^T; m = RMSNorm(h);
 *   y = h + sum_s (silu(m Wg_s^T) * (m Wu_s^T)) Wd[s]^T.
 * The projections run on the tensor cores (bf16 operands, fp32 accumulation;
 * the normalised activations feeding QKV and gate/up as bf16 hi + lo).  The
 * row-split sums add the t shard partials in ascending shard order in both
 * reduce modes, so the two modes give identical bits.
 * x, y: [T][hidden] bf16 (16-byte aligned); y32: fp32 [T][hidden] or NULL
 * (at least one of y, y32).  Requires bf16 weights (TPL_EUNSUPPORTED with
 * TPL_FP32_WEIGHTS), T <= kv->seq_cap and kv->batch_cap >= 1 (TPL_ENOMEM),
 * ws_bytes >= tpl_prefill_workspace_size(T) (TPL_EWORKSPACE).  T = 0 does
 * nothing.  Adds 2 to the plan's reduction counter. */
int tpl_prefill_layer(tpl_plan *plan, const void *packed, const tpl_kv *kv, const void *x,
                      int32_t T, void *y, float *y32, void *ws, size_t ws_bytes,
                      int32_t reduce_mode, tpl_stream stream);

/* Chunked prefill: the same layer over T tokens of one sequence whose cache
 * (batch row 0) already holds `start` tokens in slots 0..start-1.  Token i
 * sits at position start + i (its rotary angle with TPL_ROPE), attends the
 * start cached keys and the chunk's keys 0..i, and its k/v go to cache slot
 * start + i ("Tensor parallel scaling curves", "Prefill vs decode: different
 * curves": prompt tokens processed in parallel; a long prompt is taken in
 * chunks).  Requires start >= 0 and start + T <= kv->seq_cap (TPL_ENOMEM);
 * otherwise as tpl_prefill_layer, which is this call with start = 0.  A
 * chunk of one token equals a decode step at S = start. */
int tpl_prefill_chunk(tpl_plan *plan, const void *packed, const tpl_kv *kv, const void *x,
                      int32_t T, int64_t start, void *y, float *y32, void *ws, size_t ws_bytes,
                      int32_t reduce_mode, tpl_stream stream);

/* ---- the individual steps (each is one kernel launch, except where noted;
 *      the decode calls above are these in order) --------------------------- */

/* Column-parallel QKV: q [B][n_q][d] fp32; the new token's k/v go to cache
 * slot S (bf16) and, when k_new/v_new are not NULL, also to k_new/v_new
 * [B][n_kv][d] fp32 (both or neither).  With TPL_ROPE, q and k are rotated
 * to position S (a second, small kernel) before they are written out. */
int tpl_qkv(tpl_plan *plan, const void *packed, const tpl_kv *kv, const void *x, int32_t B,
            int64_t S, float *q, float *k_new, float *v_new, void *ws, size_t ws_bytes,
            tpl_stream stream);

/* Owned-head GQA decode attention over positions 0..S ("Tensor parallel
 * scaling curves", "What tensor parallelism actually splits": each shard
 * attends over the heads it owns, with no exchange).  The S cached keys are
 * split over key ranges whose partial results are combined in a fixed
 * order; the new token (position S) is taken from k_new/v_new [B][n_kv][d]
 * fp32 when given (both or neither), else from cache slot S.  o [B][n_q*d]
 * activation type.  Uses the workspace for the split partials. */
int tpl_attn_decode(tpl_plan *plan, const tpl_kv *kv, const float *q, const float *k_new,
                    const float *v_new, int32_t B, int64_t S, void *o, void *ws, size_t ws_bytes,
                    tpl_stream stream);

/* Allocation-free variant of tpl_attn_decode.  The pages have no counterpart
 * for this call; it exists for callers that cannot allocate device memory
 * themselves -- for example a plugin inside a host application whose memory
 * manager owns the whole device budget, or a latency-critical serving loop
 * that must never enter the allocator.  It takes no workspace: the split
 * partials and arrival counters live in one array of fixed size,
 * TPL_ATTN_STATIC_SCRATCH_BYTES, held in the library's static device memory
 * on every device that loads the library, until the process exits.
 *   - Same arguments as tpl_attn_decode, minus the workspace.  It runs the
 *     kernel and split geometry tpl_attn_decode chooses for the same plan,
 *     options and sizes, so the two give identical bits.
 *   - Returns TPL_ENOMEM, before launching anything, when the problem needs
 *     more scratch than that: the 256-byte-rounded sum of 4*pairs
 *     (counters), 8*pairs*n*g and 512*pairs*n*g bytes, pairs = B*n_kv, n the
 *     CTAs per pair of that geometry (the register-streamed kernel: about
 *     1024/pairs key-range splits, at least 128 keys each, four per CTA; the
 *     staged kernel: at most floor(SMs/pairs); the TMA-streamed kernel: at
 *     most ceil(min(SMs, 160)/pairs) + 1).  The 70B shapes need about 1 MB.
 *   - The first call on a device looks up the array's device address (with
 *     that device current); make that first call before any stream capture.
 *   - Every call uses the same array, and it keeps the previous call's
 *     contents; the call clears the counters it needs on `stream` first.
 *     Calls that may overlap on the GPU (other streams, other threads) race
 *     on the array and must be serialised by the caller.
 *   - Allocates nothing: no cudaMalloc, no cudaFree, no allocating library
 *     routine. */
#define TPL_ATTN_STATIC_SCRATCH_BYTES (4u * 1024u * 1024u)
int tpl_attn_decode_static(tpl_plan *plan, const tpl_kv *kv, const float *q, const float *k_new,
                           const float *v_new, int32_t B, int64_t S, void *o, tpl_stream stream);

/* Row-parallel O projection.  partials == NULL: fused, h = x + sum_s o_s
 * Wo[s]^T (fp32 [B][H]); partials != NULL: writes P[s] = o_s Wo[s]^T
 * (fp32 [t][B][H]) and leaves h untouched. */
int tpl_o_proj(tpl_plan *plan, const void *packed, const void *o, const void *x, int32_t B, float *h,
               float *partials, void *ws, size_t ws_bytes, tpl_stream stream);

/* Column-parallel gate/up with SwiGLU: act [B][F] = silu(m Wg^T) * (m Wu^T),
 * m = RMSNorm(h) [TPL_NORM] or h.  h: fp32 [B][H], or the activation type
 * when h_is_act != 0. */
int tpl_gate_up(tpl_plan *plan, const void *packed, const void *h, int32_t h_is_act, int32_t B,
                void *act, void *ws, size_t ws_bytes, tpl_stream stream);

/* Row-parallel down projection, like tpl_o_proj: fused y = h + sum_s act_s
 * Wd[s]^T (y activation type, y32 fp32 or NULL), or partials. */
int tpl_down_proj(tpl_plan *plan, const void *packed, const void *act, const float *h, int32_t B,
                  void *y, float *y32, float *partials, void *ws, size_t ws_bytes, tpl_stream stream);

/* The separate reduction: out = resid + P[0] + P[1] + ... + P[t-1] in that
 * order (resid NULL: no residual).  P fp32 [t][B][H]; resid is fp32 when
 * resid_is_f32, else the activation type; out32 fp32 (may be NULL), out_act
 * activation type (may be NULL).  Counts one reduction point. */
int tpl_reduce_partials(tpl_plan *plan, const float *P, const void *resid, int32_t resid_is_f32,
                        int32_t B, float *out32, void *out_act, tpl_stream stream);

/* The MLP pair alone (gate/up column-split, down row-split; flags decide the
 * norm and the residual): y = [x +] sum_s (silu(a Wg_s^T) * (a Wu_s^T)) Wd[s]^T,
 * a = RMSNorm(x) [TPL_NORM] or x.  "Tensor Parallelism Fundamentals",
 * "Mechanics of Matrix Slicing" (the feed-forward example). */
int tpl_mlp_block(tpl_plan *plan, const void *packed, const void *x, int32_t B, void *y, float *y32,
                  void *ws, size_t ws_bytes, int32_t reduce_mode, tpl_stream stream);

/* ---- diagnostics -------------------------------------------------------- */

/* Reduction points launched through this plan since creation/reset. */
int64_t tpl_reduction_count(const tpl_plan *plan);

/* Host: the number of kernels a decode call launches for B tokens in the
 * given reduce mode: tpl_decode_layer with n_layers = 1, tpl_decode_stack
 * over n_layers layers (the projections' kernel family, the operand kernels
 * of the tensor-core projections that the fused row-parallel kernels do not
 * already cover, the rotation, the separate reductions). */
int tpl_decode_kernel_count(const tpl_plan *plan, int32_t B, int32_t reduce_mode, int32_t n_layers,
                            int32_t *count);
void tpl_reset_counters(tpl_plan *plan);

/* Synchronise `stream`, read and clear the device error word of the current
 * device.  TPL_OK, TPL_EDEVICE (a kernel recorded an inconsistency) or
 * TPL_ECUDA (the stream reported an error). */
int tpl_last_device_error(const tpl_plan *plan, tpl_stream stream);

/* Timeline trace (the diagnostic build of the library, compiled with
 * -DTPL_TRACE; the ordinary build returns TPL_EUNSUPPORTED and writes 0 to
 * *n_records).  Each decode kernel appends one record per CTA: a tag (1 QKV,
 * 2 attention, 3 O, 4 gate/up, 5 down, 6 operand kernel), the CTA index, its
 * SM, the grid size, and four global-timer values in ns (entry, dependency
 * wait passed, main loop done, exit; 0 where a kernel takes no such mark).
 * records: host array of max_records records of 48 bytes (4 x uint32 then 4
 * x uint64).  Synchronises the device, copies up to max_records of the
 * records taken since the last read and starts a new trace. */
int tpl_trace_read(void *records, int32_t max_records, int32_t *n_records);

/* Static description of a status code. */
const char *tpl_status_string(int status);

#if defined(__GNUC__)
#pragma GCC visibility pop
#endif
#ifdef __cplusplus
}
#endif
#endif /* TPL_H */
