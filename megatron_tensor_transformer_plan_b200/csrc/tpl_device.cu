// Kernels and C-ABI entry points of libtpl (one translation unit, so the
// device error word is a plain __device__ variable).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstring>

#include "tpl_attn.cuh"
#include "tpl_attn_tma.cuh"
#include "tpl_common.cuh"
#include "tpl_gemv.cuh"
#include "tpl_gemv_tc.cuh"
#include "tpl_internal.h"
#include "tpl_norm.cuh"
#include "tpl_rope.cuh"
#include "tpl_tma.h"

namespace tpl {

// out = resid + ((P[0] + P[1]) + ... + P[t-1]), the separate form of the
// row-split sum ("Tensor parallel scaling curves": the all-reduce after the
// output and down projections).  Same order and operations as the fused
// epilogue of gemv_kernel, hence identical bits.
__global__ void reduce_partials_kernel(const float *__restrict__ P, int t, int64_t n, const void *resid,
                                       int resid_f32, float *out32, void *out_act, int act_f32) {
    pdl_wait();
    pdl_trigger();
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        float acc = P[i];
        for (int s = 1; s < t; ++s) acc = acc + P[(int64_t)s * n + i];
        if (resid) acc = load_act(resid, resid_f32, i) + acc;
        if (out32) out32[i] = acc;
        if (out_act) store_act(out_act, act_f32, i, acc);
    }
}

__global__ void fill_f32_kernel(float *p, int64_t n, float v) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
        p[i] = v;
}

namespace {

// Launch with programmatic dependent launch enabled: the kernel may start
// while the previous kernel on the stream drains; every kernel here waits
// (griddepcontrol.wait) before touching data a previous kernel wrote.
template <typename... KA, typename... A>
cudaError_t launch_pdl(void (*kern)(KA...), dim3 grid, int block, size_t smem, cudaStream_t st, A &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<A>(args)...);
}

bool g_attr_done[64][8];

// Preferred carve-out of a kernel with static shared memory only: the share
// of the SM's shared memory that its resident CTAs need (as many as fit by
// registers and threads), rounded up by the driver to a supported size.
template <typename K>
cudaError_t set_fit_carveout(K kern, int threads) {
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, kern);
    int dev = 0, blocks = 0, smem_sm = 0;
    if (e == cudaSuccess) e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
    if (e == cudaSuccess) e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&blocks, kern, threads, 0);
    if (e != cudaSuccess) return e;
    if (blocks < 1 || smem_sm <= 0) return cudaSuccess;  // keep the default
    const long need = (long)blocks * ((long)fa.sharedSizeBytes + 1024);  // 1 KB reserved per CTA
    const int pct = (int)std::min<long>(100, (need * 100 + smem_sm - 1) / smem_sm);
    return cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, pct);
}

// The mma.sync projections stream their weights through registers, and a
// load in flight holds L1 staging space: they ask for the smallest shared-
// memory carve-out that fits them (the rest of the 256 KB is L1).  Without
// the preference an SM keeps the carve-out of the kernel before (228 KB after
// a staged attention of 204 KB), which left 28 KB of L1 and ran every
// projection of the 7B layer about 50% slower.
template <int MODE, bool BIG>
cudaError_t set_smem_attr() {
    cudaError_t e = cudaFuncSetAttribute(gemv_kernel<MODE, BIG>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         227 * 1024);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(gemv_kernel<MODE, BIG>, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 (int)cudaSharedmemCarveoutMaxL1);
    return e;
}

int prepare_gemv(int mode, bool big) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return TPL_ECUDA;
    const int slot = mode * 2 + (big ? 1 : 0);
    if (!g_attr_done[dev][slot]) {
        cudaError_t e;
        switch (slot) {
            case 0: e = set_smem_attr<0, false>(); break;
            case 1: e = set_smem_attr<0, true>(); break;
            case 2: e = set_smem_attr<1, false>(); break;
            case 3: e = set_smem_attr<1, true>(); break;
            case 4: e = set_smem_attr<2, false>(); break;
            case 5: e = set_smem_attr<2, true>(); break;
            case 6: e = set_smem_attr<3, false>(); break;
            default: e = set_smem_attr<3, true>(); break;
        }
        if (e != cudaSuccess) return TPL_ECUDA;
        g_attr_done[dev][slot] = true;
    }
    return TPL_OK;
}

int cuda_rc(cudaError_t e) { return e == cudaSuccess ? TPL_OK : TPL_ECUDA; }

bool al16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

struct Ctx {
    tpl_plan *p;
    char *ws;
    WsLayout L;
    cudaStream_t st;
    int B;
    int64_t S;
    // the tensor-core projections' operand (workspace xs) already holds the
    // split x * gamma_attn of this layer's input (written by the previous
    // layer's down projection), or h * gamma_mlp (written by O)
    bool xs_holds_x = false, xs_holds_h = false;
    const float *next_gamma = nullptr;  // gamma_attn of the next layer of a stack
    bool has_next = false;
};

int make_ctx(tpl_plan *p, void *ws, size_t ws_bytes, int B, int64_t S, tpl_stream stream, Ctx *c) {
    if (!p || !ws || !al16(ws)) return TPL_EINVAL;
    if (B < 1 || S < 0) return TPL_EINVAL;
    if (B > (p->f32 ? kMaxBatchCuda : kMaxBatch)) return TPL_EUNSUPPORTED;
    int rc = ws_layout(p, B, S, &c->L);
    if (rc != TPL_OK) return rc;
    if (ws_bytes < c->L.total) return TPL_EWORKSPACE;
    c->p = p;
    c->ws = static_cast<char *>(ws);
    c->st = static_cast<cudaStream_t>(stream);
    c->B = B;
    c->S = S;
    return TPL_OK;
}

int check_kv(const tpl_kv *kv, int B, int64_t S) {
    if (!kv || !kv->k || !kv->v || !al16(kv->k) || !al16(kv->v)) return TPL_EINVAL;
    if (kv->batch_cap < B || kv->seq_cap <= S || S < 0) return TPL_ENOMEM;
    return TPL_OK;
}

int gemv_launch(Ctx &c, GemvArgs &a, int N, int nseg, int Kseg, int op) {
    tpl_plan *p = c.p;
    a.trace_row_tag = op == OP_O ? TR_O : TR_DOWN;
    if (c.B > kMaxBatchCuda) return TPL_EUNSUPPORTED;
    const int sms = num_sms_current();
    if (sms <= 0) return TPL_ECUDA;
    // The Q projection feeds a softmax and gate/up feeds SwiGLU: carry their
    // normalised activations as bf16 hi + lo.
    const int mode = p->f32 ? 1 : (p->gemv_mode == 2 ? 2 : ((op == OP_QKV || op == OP_GU) ? 3 : 0));  // modes 0, 4
    int rc = gemv_geom(N, nseg, Kseg, c.B, p->f32 ? 4 : 2, sms, &a.g, mode == 3 ? 2 : 1);
    if (rc != TPL_OK) return rc;
    const bool big = c.B > 8;
    rc = prepare_gemv(mode, big);
    if (rc != TPL_OK) return rc;
    a.B = c.B;
    a.gp = reinterpret_cast<float *>(c.ws + c.L.gp);
    a.tickets = reinterpret_cast<unsigned *>(c.ws + c.L.tickets) + kTicketGemv + 512 * op;
    const int grid = a.g.rb * a.g.ksplit;
    const size_t sm = a.g.smem;
    cudaError_t e;
    switch (mode * 2 + (big ? 1 : 0)) {
        case 0: e = launch_pdl(gemv_kernel<0, false>, grid, kGemvThreads, sm, c.st, a); break;
        case 1: e = launch_pdl(gemv_kernel<0, true>, grid, kGemvThreads, sm, c.st, a); break;
        case 2: e = launch_pdl(gemv_kernel<1, false>, grid, kGemvThreads, sm, c.st, a); break;
        case 3: e = launch_pdl(gemv_kernel<1, true>, grid, kGemvThreads, sm, c.st, a); break;
        case 4: e = launch_pdl(gemv_kernel<2, false>, grid, kGemvThreads, sm, c.st, a); break;
        case 5: e = launch_pdl(gemv_kernel<2, true>, grid, kGemvThreads, sm, c.st, a); break;
        case 6: e = launch_pdl(gemv_kernel<3, false>, grid, kGemvThreads, sm, c.st, a); break;
        default: e = launch_pdl(gemv_kernel<3, true>, grid, kGemvThreads, sm, c.st, a); break;
    }
    return cuda_rc(e);
}

GemvArgs base_args(const tpl_plan *p) {
    GemvArgs a;
    std::memset(&a, 0, sizeof(a));
    a.act_f32 = p->f32 ? 1 : 0;
    a.eps = p->d.rms_eps;
    a.hd = p->d.head_dim;
    return a;
}

// ---- tensor-core decode projections (TPL_OPT_GEMV_MODE 3) -----------------

bool g_gt_attr[64][8];

template <int NX, bool SPLIT>
int gt_go(int slot, GemvTcArgs &a, cudaStream_t st) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return TPL_ECUDA;
    if (!g_gt_attr[dev][slot]) {
        if (cudaFuncSetAttribute(gemv_tc_kernel<NX, SPLIT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 GemvTcSmem<NX, SPLIT>::BYTES) != cudaSuccess)
            return TPL_ECUDA;
        g_gt_attr[dev][slot] = true;
    }
    const int sms = num_sms_current();
    if (sms <= 0) return TPL_ECUDA;
    const int64_t G = std::min<int64_t>(std::min<int64_t>(sms, a.U), kGemvTcMaxCtas);
    return cuda_rc(
        launch_pdl(gemv_tc_kernel<NX, SPLIT>, (int)G, kGtThreads, (size_t)GemvTcSmem<NX, SPLIT>::BYTES, st, a));
}

// A layer of at least 1 GiB of bf16 weights (the 70B shape; the 7B layer is
// 0.4 GiB): the decode kernels' choices below differ by layer size.
bool large_layer(const tpl_plan *p) {
    const tpl_dims &d = p->d;
    const int64_t layer_params = (int64_t)(d.n_q_heads + 2 * d.n_kv_heads) * d.head_dim * d.hidden +
                                 (int64_t)d.hidden * d.n_q_heads * d.head_dim + 3 * (int64_t)d.ffn * d.hidden;
    return layer_params * 2 >= (1ll << 30);
}

// Fill the geometry, the weight map (2-D column-parallel rows or 3-D per-shard
// blocks) and the activation map, then launch.
int gemv_tc_run(Ctx &c, GemvTcArgs &a, int op, bool split, const void *W, int64_t ld, int64_t N, int nseg,
                int64_t blk, const void *X, int64_t Kx, int64_t x_rows, int x_seg_stride) {
    if (c.B > kGtMaxB) return TPL_EUNSUPPORTED;
    // On small layers 9 to 16 tokens unsplit take the split form's 32 columns
    // (the upper 16 read as zero rows), so that all four projections run one
    // kernel binary (7B layer, 16 tokens: 224 -> 220 us); on large layers the
    // extra operand bytes per stage cost more than the shared code saves
    const bool widen = !split && c.B > 8 && c.B <= 16 && !large_layer(c.p);
    const int nx = widen ? 32 : gt_nx(c.B, split);
    a.B = c.B;
    a.N = (int)N;
    a.tiles = (int)((N + kGtRows - 1) / kGtRows);
    if (a.tiles > kGemvTcMaxTiles) return TPL_EUNSUPPORTED;
    a.nseg = nseg;
    a.kbs = (int)(ld / kGtK);
    a.U = (int64_t)a.tiles * a.nseg * a.kbs;
    a.x_seg_stride = x_seg_stride;
    a.w3d = nseg > 1 ? 1 : 0;
    int rc = a.w3d ? make_map(&a.tm_w, W, ld, N, ld * 2, kGtK, kGtRows, nseg, blk)
                   : make_map(&a.tm_w, W, ld, N, ld * 2, kGtK, kGtRows);
    if (rc == TPL_OK) rc = make_map(&a.tm_x, X, Kx, x_rows, Kx * 2, kGtK, nx);
    if (rc != TPL_OK) return rc;
    a.gpart = reinterpret_cast<float *>(c.ws + c.L.gpart);
    a.gstride = gt_stride(c.B);
    a.tickets = reinterpret_cast<unsigned *>(c.ws + c.L.tickets) + kTicketGemv + 512 * op;
    a.xsplit = split ? 1 : 0;
    // up to 8 tokens the split and unsplit forms share one kernel (see
    // gt_load_chunk); from 9 tokens the split form needs more columns anyway
    if (nx == 16 && (split || c.B <= 8)) return gt_go<16, true>(0, a, c.st);
    if (split || widen) {
        switch (nx) {
            case 32: return gt_go<32, true>(1, a, c.st);
            case 64: return gt_go<64, true>(2, a, c.st);
            default: return gt_go<128, true>(3, a, c.st);
        }
    }
    switch (nx) {
        case 16: return gt_go<16, false>(4, a, c.st);
        case 32: return gt_go<32, false>(5, a, c.st);
        default: return gt_go<64, false>(6, a, c.st);
    }
}

// TPL_OPT_GEMV_MODE 4 (the default for bf16 plans): one kernel family for all
// four projections of a layer, the one that measured faster on B200 (layers
// that mix the two families measured slower than either): tcgen05 on layers
// of at least 1 GiB of weights at any token count (70B layer, one token: 304
// against 312 us) and from 7 tokens on any layer, mma.sync for up to 6 tokens
// on small layers (7B layer at t = 1, one token: 99.9 against 115.2 us; six:
// 155.0 against 158.1; seven: 161.3 against 160.2).
// Beyond 16 tokens (any mode) only the tcgen05 kernel applies.
bool use_tc(const tpl_plan *p, int op, int B) {
    (void)op;
    if (p->f32) return false;
    if (B > kMaxBatchCuda) return true;  // beyond the mma.sync kernel's 16 tokens
    if (p->gemv_mode == 3) return true;
    if (p->gemv_mode != 4) return false;
    return large_layer(p) || B >= 7;
}

GemvTcArgs gt_args(const tpl_plan *p) {
    GemvTcArgs a;
    std::memset(&a, 0, sizeof(a));
    a.hd = p->d.head_dim;
    return a;
}

// The tensor-core projections' activation operand [NX][hidden] in the
// workspace: x * gamma (x without TPL_NORM) as bf16 hi rows 0..B-1 and lo
// rows NX/2..; the RMSNorm factor 1/rms is applied by the projection.
int run_scale_split(Ctx &c, const void *x, int x_f32, const float *gamma) {
    tpl_plan *p = c.p;
    auto *xs = reinterpret_cast<__nv_bfloat16 *>(c.ws + c.L.xs);
    const int half = gt_nx(c.B, true) / 2;
    const int H = p->d.hidden;
    const dim3 grid((unsigned)((H / 8 + 255) / 256), (unsigned)c.B);
    return cuda_rc(launch_pdl(scale_split_kernel, grid, 256, 0, c.st, x, x_f32,
                              (p->d.flags & TPL_NORM) ? gamma : nullptr, H, xs, half));
}

// The folded RMSNorm of a column-parallel projection: 1/rms of src's rows.
void set_rms(const tpl_plan *p, GemvTcArgs &a, const void *src, int src_f32) {
    if (!(p->d.flags & TPL_NORM)) return;
    a.rms_src = src;
    a.rms_f32 = src_f32;
    a.rms_len = p->d.hidden;
    a.rms_eps = p->d.rms_eps;
}

int run_qkv_tc(Ctx &c, const char *packed, const tpl_kv *kv, const void *x, float *q, float *knew, float *vnew) {
    tpl_plan *p = c.p;
    if (!c.xs_holds_x) {
        int rc = run_scale_split(c, x, 0, reinterpret_cast<const float *>(packed + p->off_g1));
        if (rc != TPL_OK) return rc;
    }
    c.xs_holds_x = false;
    GemvTcArgs a = gt_args(p);
    set_rms(p, a, x, 0);
    a.epi = GT_QKV;
    a.q = q;
    a.knew = knew;
    a.vnew = vnew;
    a.kc = static_cast<__nv_bfloat16 *>(kv->k);
    a.vc = static_cast<__nv_bfloat16 *>(kv->v);
    a.rps = p->qkv_rows_s;
    a.nq = p->d.n_q_heads;
    a.nq_s = p->nq_s;
    a.nkv_s = p->nkv_s;
    a.batch_cap = kv->batch_cap;
    a.S = c.S;
    a.seq_cap = kv->seq_cap;
    const int64_t H = p->d.hidden;
    return gemv_tc_run(c, a, OP_QKV, true, packed + p->off_qkv, p->ld_h, (int64_t)p->t * p->qkv_rows_s, 1, 0,
                       c.ws + c.L.xs, H, gt_nx(c.B, true), 0);
}

int run_gu_tc(Ctx &c, const char *packed, const void *h, int h_is_act, void *act) {
    tpl_plan *p = c.p;
    if (!c.xs_holds_h) {
        int rc = run_scale_split(c, h, h_is_act ? 0 : 1, reinterpret_cast<const float *>(packed + p->off_g2));
        if (rc != TPL_OK) return rc;
    }
    c.xs_holds_h = false;
    GemvTcArgs a = gt_args(p);
    set_rms(p, a, h, h_is_act ? 0 : 1);
    a.epi = GT_GU;
    a.out_act = act;
    const int64_t H = p->d.hidden;
    return gemv_tc_run(c, a, OP_GU, true, packed + p->off_gu, p->ld_h, (int64_t)p->t * 2 * p->F_s, 1, 0,
                       c.ws + c.L.xs, H, gt_nx(c.B, true), 0);
}

// Row-parallel O (K slice of shard s: columns s*nq_s*d of o) or down (s*F_s of act).
// With xs_gamma_or_mark set (fused mode inside a layer or a stack), the
// epilogue also writes the next column-parallel projection's operand:
// xs = split(out * gamma), gamma = xs_gamma (NULL without TPL_NORM).
int run_row_tc(Ctx &c, const char *packed, int op, const void *x, const void *resid, int resid_f32, float *out32,
               void *out_act, float *partials, bool write_xs = false, const float *xs_gamma = nullptr) {
    tpl_plan *p = c.p;
    GemvTcArgs a = gt_args(p);
    a.trace_row_tag = op == OP_O ? TR_O : TR_DOWN;
    if (partials) {
        a.epi = GT_ROW_PARTIAL;
        a.partials = partials;
    } else {
        a.epi = GT_ROW;
        a.resid = resid;
        a.resid_f32 = resid_f32;
        a.out32 = out32;
        a.out_act = out_act;
        if (write_xs) {
            a.xs_out = reinterpret_cast<__nv_bfloat16 *>(c.ws + c.L.xs);
            a.xs_gamma = (p->d.flags & TPL_NORM) ? xs_gamma : nullptr;
            a.xs_half = gt_nx(c.B, true) / 2;
        }
    }
    const bool is_o = op == OP_O;
    const int64_t Ks = is_o ? (int64_t)p->nq_s * p->d.head_dim : p->F_s;
    const int64_t ld = is_o ? p->ld_o : p->ld_f;
    const int64_t blk = is_o ? p->blk_o : p->blk_d;
    const char *W = packed + (is_o ? p->off_o : p->off_d);
    if (p->t == 1) {
        // one shard: a single 2-D block
        return gemv_tc_run(c, a, op, false, W, ld, p->d.hidden, 1, 0, x, Ks, c.B, 0);
    }
    return gemv_tc_run(c, a, op, false, W, ld, p->d.hidden, p->t, blk, x, (int64_t)p->t * Ks, c.B, (int)Ks);
}

int run_qkv_proj(Ctx &c, const char *packed, const tpl_kv *kv, const void *x, float *q, float *knew,
                 float *vnew) {
    tpl_plan *p = c.p;
    if (use_tc(p, OP_QKV, c.B)) return run_qkv_tc(c, packed, kv, x, q, knew, vnew);
    GemvArgs a = base_args(p);
    a.W = packed + p->off_qkv;
    a.blk_r = p->blk_qkv;
    a.rps = p->qkv_rows_s;
    a.ldw = p->ld_h;
    a.x = x;
    a.x_f32 = p->f32;
    a.ldx = p->d.hidden;
    a.norm = (p->d.flags & TPL_NORM) ? 1 : 0;
    a.gamma = reinterpret_cast<const float *>(packed + p->off_g1);
    a.epi = EPI_QKV;
    a.q = q;
    a.knew = knew;
    a.vnew = vnew;
    a.kc = static_cast<__nv_bfloat16 *>(kv->k);
    a.vc = static_cast<__nv_bfloat16 *>(kv->v);
    a.nq = p->d.n_q_heads;
    a.nq_s = p->nq_s;
    a.nkv_s = p->nkv_s;
    a.batch_cap = kv->batch_cap;
    a.S = c.S;
    a.seq_cap = kv->seq_cap;
    return gemv_launch(c, a, p->t * p->qkv_rows_s, 1, p->d.hidden, OP_QKV);
}

// The QKV step: the projection, then (TPL_ROPE) the rotation of q and the new
// k to position S, which needs the unrounded keys: without caller buffers
// the workspace's copies are used.
int run_qkv(Ctx &c, const char *packed, const tpl_kv *kv, const void *x, float *q, float *knew, float *vnew) {
    tpl_plan *p = c.p;
    if (p->rope && !knew) {
        knew = reinterpret_cast<float *>(c.ws + c.L.knew);
        vnew = reinterpret_cast<float *>(c.ws + c.L.vnew);
    }
    int rc = run_qkv_proj(c, packed, kv, x, q, knew, vnew);
    if (rc != TPL_OK || !p->rope) return rc;
    RopeArgs r;
    std::memset(&r, 0, sizeof(r));
    r.q = q;
    r.knew = knew;
    r.kc = static_cast<__nv_bfloat16 *>(kv->k);
    r.B = c.B;
    r.nq = p->d.n_q_heads;
    r.nkv = p->d.n_kv_heads;
    r.nkv_s = p->nkv_s;
    r.batch_cap = kv->batch_cap;
    r.seq_cap = kv->seq_cap;
    r.pos = c.S;
    std::memcpy(r.theta, p->rope_theta, sizeof(r.theta));
    const int64_t heads = (int64_t)c.B * (r.nq + r.nkv);
    const int64_t grid = (heads + kRopeThreads / 64 - 1) / (kRopeThreads / 64);
    return cuda_rc(launch_pdl(rope_decode_kernel, (int)grid, kRopeThreads, 0, c.st, r));
}

bool g_stg_attr[64];

// Which decode attention kernel runs and its split geometry.
//   TPL_OPT_DECODE_ATTN 0 (default): the TMA-streamed kernel for groups of at
//     most 8 heads when the pairs fit one wave of SMs and each has at least
//     kAttnTmaMinKeys cached keys (70B layer, batch 16, 8192 keys: 96.8 us
//     against 104.9); else the staged kernel for groups of at most 8 heads
//     with at least two CTAs per pair in one wave; else the register-streamed
//     kernel (with one CTA per pair its finer splits win);
//   1: the register-streamed kernel;
//   2: the TMA-streamed kernel (groups of at most 8 heads, at least one
//      cached key), else as 0.
enum { ATTN_REG = 0, ATTN_STAGED = 1, ATTN_TMA = 2 };
constexpr int64_t kAttnTmaMinKeys = 8192;
int attn_select(const tpl_plan *p, int B, int64_t keys, AttnGeom *g, int *kind) {
    const int sms = num_sms_current();
    if (sms <= 0) return TPL_ECUDA;
    const bool tma_ok = p->g <= kAmMaxG && keys >= 1 && keys <= 0x7fffffffll;
    const bool tma_auto = p->attn_decode_mode == 0 && B * p->d.n_kv_heads <= sms && keys >= kAttnTmaMinKeys;
    if (tma_ok && (p->attn_decode_mode == 2 || tma_auto)) {
        attn_geom_tma(B, p->d.n_kv_heads, keys, sms, g);
        *kind = ATTN_TMA;
    } else if (p->attn_decode_mode != 1 && p->g <= 8 && 2 * B * p->d.n_kv_heads <= sms) {
        attn_geom_staged(B, p->d.n_kv_heads, keys, sms, g);
        *kind = ATTN_STAGED;
    } else {
        attn_geom(B, p->d.n_kv_heads, keys, g);
        *kind = ATTN_REG;
    }
    if (g->pairs > kMaxPairs) return TPL_EUNSUPPORTED;
    return TPL_OK;
}

// CTA partials per pair the chosen kernel writes (sizes its scratch).
int attn_cpp(const AttnGeom &g, int kind) {
    return kind == ATTN_TMA ? g.cpp_max : g.nsplit / (kind == ATTN_STAGED ? kAttnStgWarps : kAttnWarps);
}

bool g_am_attr[64];
bool g_reg_attr[64];

// Fill the launch arguments (everything except the scratch pointers) and
// launch the kernel attn_select chose.
int attn_launch(const tpl_plan *p, const tpl_kv *kv, const float *q, const float *knew, const float *vnew, int B,
                int64_t keys, void *o, const AttnGeom &g, int kind, unsigned *tickets, float *part_ml,
                float *part_o, cudaStream_t st) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return TPL_ECUDA;
    const float scale_log2 = 1.4426950408889634f / sqrtf((float)p->d.head_dim);
    if (kind == ATTN_TMA) {
        AttnTmaArgs a;
        std::memset(&a, 0, sizeof(a));
        const uint64_t sb = (uint64_t)p->t * kv->batch_cap;
        int rc = make_kv_map(&a.tm_k, kv->k, (uint64_t)keys, (uint64_t)p->nkv_s, sb, (uint64_t)kv->seq_cap, kAmKeys);
        if (rc == TPL_OK)
            rc = make_kv_map(&a.tm_v, kv->v, (uint64_t)keys, (uint64_t)p->nkv_s, sb, (uint64_t)kv->seq_cap, kAmKeys);
        if (rc != TPL_OK) return rc;
        a.q = q;
        a.B = B;
        a.nq = p->d.n_q_heads;
        a.nkv_s = p->nkv_s;
        a.g = p->g;
        a.batch_cap = kv->batch_cap;
        a.keys = (int)keys;
        a.nb = g.nb;
        a.U = (int64_t)g.pairs * g.nb;
        a.k_new = knew;
        a.v_new = vnew;
        a.scale_log2 = scale_log2;
        a.part_o = part_o;
        a.part_ml = part_ml;
        a.cpp_max = g.cpp_max;
        a.tickets = tickets;
        a.o = o;
        a.o_f32 = p->f32;
        if (!g_am_attr[dev]) {
            if (cudaFuncSetAttribute(attn_decode_tma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)kAmSmem) != cudaSuccess)
                return TPL_ECUDA;
            g_am_attr[dev] = true;
        }
        return cuda_rc(launch_pdl(attn_decode_tma_kernel, g.grid, kAmThreads, kAmSmem, st, a));
    }
    AttnArgs a;
    std::memset(&a, 0, sizeof(a));
    a.q = q;
    a.kc = static_cast<const __nv_bfloat16 *>(kv->k);
    a.vc = static_cast<const __nv_bfloat16 *>(kv->v);
    a.seq_cap = kv->seq_cap;
    a.batch_cap = kv->batch_cap;
    a.B = B;
    a.nq = p->d.n_q_heads;
    a.nkv_s = p->nkv_s;
    a.g = p->g;
    a.keys = keys;
    a.k_new = knew;
    a.v_new = vnew;
    a.nsplit = g.nsplit;
    a.kps = g.kps;
    a.scale_log2 = scale_log2;
    a.part_o = part_o;
    a.part_ml = part_ml;
    a.tickets = tickets;
    a.o = o;
    a.o_f32 = p->f32;
    const int grid = g.pairs * attn_cpp(g, kind);
    if (kind == ATTN_STAGED) {
        if (!g_stg_attr[dev]) {
            if (cudaFuncSetAttribute(attn_decode_staged_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)kStgSmem) != cudaSuccess)
                return TPL_ECUDA;
            g_stg_attr[dev] = true;
        }
        return cuda_rc(launch_pdl(attn_decode_staged_kernel, grid, kAttnStgWarps * 32, kStgSmem, st, a));
    }
    if (!g_reg_attr[dev]) {
        // register-streamed K/V: as for the mma.sync projections, a carve-out
        // just large enough for the CTAs that fit an SM by registers, so that
        // the loads in flight have L1 to land in (the smallest carve-out
        // would cut the resident CTAs instead)
        if (set_fit_carveout(attn_decode_kernel<true>, kAttnWarps * 32) != cudaSuccess ||
            set_fit_carveout(attn_decode_kernel<false>, kAttnWarps * 32) != cudaSuccess)
            return TPL_ECUDA;
        g_reg_attr[dev] = true;
    }
    return cuda_rc(p->g <= 8 ? launch_pdl(attn_decode_kernel<true>, grid, kAttnWarps * 32, 0, st, a)
                              : launch_pdl(attn_decode_kernel<false>, grid, kAttnWarps * 32, 0, st, a));
}

int run_attn(Ctx &c, const tpl_kv *kv, const float *q, const float *knew, const float *vnew, void *o) {
    tpl_plan *p = c.p;
    const int64_t keys = knew ? c.S : c.S + 1;
    AttnGeom g;
    int kind = 0;
    int rc = attn_select(p, c.B, keys, &g, &kind);
    if (rc != TPL_OK) return rc;
    return attn_launch(p, kv, q, knew, vnew, c.B, keys, o, g, kind,
                       reinterpret_cast<unsigned *>(c.ws + c.L.tickets) + kTicketAttn,
                       reinterpret_cast<float *>(c.ws + c.L.part_ml), reinterpret_cast<float *>(c.ws + c.L.part_o),
                       c.st);
}

// Row-parallel O projection: fused (partials == NULL) or partial output.
// With `chain` (inside a layer, fused mode) the tensor-core kernel also
// writes gate/up's operand h * gamma_mlp.
int run_o(Ctx &c, const char *packed, const void *o, const void *resid, float *h, float *partials,
          bool chain = false) {
    tpl_plan *p = c.p;
    if (use_tc(p, OP_O, c.B)) {
        const bool wx = chain && !partials;
        int rc = run_row_tc(c, packed, OP_O, o, resid, 0, h, nullptr, partials, wx,
                            reinterpret_cast<const float *>(packed + p->off_g2));
        if (rc == TPL_OK && !partials) p->reductions.fetch_add(1);
        if (rc == TPL_OK && wx) c.xs_holds_h = true;
        return rc;
    }
    GemvArgs a = base_args(p);
    a.W = packed + p->off_o;
    a.blk_s = p->blk_o;
    a.rps = p->d.hidden;
    a.ldw = p->ld_o;
    a.x = o;
    a.x_f32 = p->f32;
    a.ldx = p->d.n_q_heads * p->d.head_dim;
    if (partials) {
        a.epi = EPI_ROW_PARTIAL;
        a.partials = partials;
    } else {
        a.epi = EPI_ROW;
        a.resid = resid;
        a.resid_f32 = p->f32;
        a.out32 = h;
    }
    int rc = gemv_launch(c, a, p->d.hidden, p->t, p->nq_s * p->d.head_dim, OP_O);
    if (rc == TPL_OK && !partials) p->reductions.fetch_add(1);
    return rc;
}

int run_gu(Ctx &c, const char *packed, const void *h, int h_is_act, void *act) {
    tpl_plan *p = c.p;
    if (use_tc(p, OP_GU, c.B)) return run_gu_tc(c, packed, h, h_is_act, act);
    GemvArgs a = base_args(p);
    a.W = packed + p->off_gu;
    a.blk_r = p->blk_gu;
    a.rps = 2 * p->F_s;
    a.ldw = p->ld_h;
    a.x = h;
    a.x_f32 = h_is_act ? p->f32 : 1;
    a.ldx = p->d.hidden;
    a.norm = (p->d.flags & TPL_NORM) ? 1 : 0;
    a.gamma = reinterpret_cast<const float *>(packed + p->off_g2);
    a.epi = EPI_GU;
    a.out_act = act;
    return gemv_launch(c, a, p->t * 2 * p->F_s, 1, p->d.hidden, OP_GU);
}

// With `chain` (a stack layer followed by another, fused mode) the
// tensor-core kernel also writes the next layer's QKV operand y * gamma_attn.
int run_down(Ctx &c, const char *packed, const void *act, const void *resid, int resid_f32, void *y, float *y32,
             float *partials, bool chain = false) {
    tpl_plan *p = c.p;
    if (use_tc(p, OP_DOWN, c.B)) {
        const bool wx = chain && !partials && y && c.has_next;
        int rc = run_row_tc(c, packed, OP_DOWN, act, resid, resid_f32, y32, y, partials, wx, c.next_gamma);
        if (rc == TPL_OK && !partials) p->reductions.fetch_add(1);
        if (rc == TPL_OK && wx) c.xs_holds_x = true;
        return rc;
    }
    GemvArgs a = base_args(p);
    a.W = packed + p->off_d;
    a.blk_s = p->blk_d;
    a.rps = p->d.hidden;
    a.ldw = p->ld_f;
    a.x = act;
    a.x_f32 = p->f32;
    a.ldx = p->d.ffn;
    if (partials) {
        a.epi = EPI_ROW_PARTIAL;
        a.partials = partials;
    } else {
        a.epi = EPI_ROW;
        a.resid = resid;
        a.resid_f32 = resid_f32;
        a.out32 = y32;
        a.out_act = y;
    }
    int rc = gemv_launch(c, a, p->d.hidden, p->t, p->F_s, OP_DOWN);
    if (rc == TPL_OK && !partials) p->reductions.fetch_add(1);
    return rc;
}

int run_reduce(tpl_plan *p, cudaStream_t st, const float *P, const void *resid, int resid_f32, int B, float *out32,
               void *out_act) {
    const int64_t n = (int64_t)B * p->d.hidden;
    const int grid = (int)std::min<int64_t>((n + 255) / 256, 4 * 148);
    int rc = cuda_rc(launch_pdl(reduce_partials_kernel, grid, 256, 0, st, P, p->t, n, resid, resid_f32, out32, out_act,
                                p->f32 ? 1 : 0));
    if (rc == TPL_OK) p->reductions.fetch_add(1);
    return rc;
}

// One decode layer: x (activation type) -> y (activation type) [+ y32].
int decode_layer(Ctx &c, const char *packed, const tpl_kv *kv, const void *x, void *y, float *y32, int mode) {
    tpl_plan *p = c.p;
    const bool resid = (p->d.flags & TPL_RESIDUAL) != 0;
    float *q = reinterpret_cast<float *>(c.ws + c.L.q);
    void *o = c.ws + c.L.o;
    float *h = reinterpret_cast<float *>(c.ws + c.L.h);
    void *act = c.ws + c.L.act;
    float *P = reinterpret_cast<float *>(c.ws + c.L.P);
    float *knew = reinterpret_cast<float *>(c.ws + c.L.knew);
    float *vnew = reinterpret_cast<float *>(c.ws + c.L.vnew);
    int rc = run_qkv(c, packed, kv, x, q, knew, vnew);
    if (rc == TPL_OK) rc = run_attn(c, kv, q, knew, vnew, o);
    if (rc == TPL_OK) {
        if (mode == TPL_REDUCE_FUSED) {
            rc = run_o(c, packed, o, resid ? x : nullptr, h, nullptr, true);
        } else {
            rc = run_o(c, packed, o, nullptr, nullptr, P);
            if (rc == TPL_OK) rc = run_reduce(p, c.st, P, resid ? x : nullptr, p->f32, c.B, h, nullptr);
        }
    }
    if (rc == TPL_OK) rc = run_gu(c, packed, h, 0, act);
    if (rc == TPL_OK) {
        if (mode == TPL_REDUCE_FUSED) {
            rc = run_down(c, packed, act, resid ? h : nullptr, 1, y, y32, nullptr, true);
        } else {
            rc = run_down(c, packed, act, nullptr, 1, nullptr, nullptr, P);
            if (rc == TPL_OK) rc = run_reduce(p, c.st, P, resid ? h : nullptr, 1, c.B, y32, y);
        }
    }
    return rc;
}

}  // namespace
}  // namespace tpl

// The prefill path: its kernels and host orchestration use the helpers above.
#include "tpl_prefill.cuh"

using namespace tpl;

extern "C" {

int tpl_workspace_init(const tpl_plan *plan, void *ws, size_t ws_bytes, tpl_stream stream) {
    if (!plan || !ws) return TPL_EINVAL;
    if (ws_bytes < sizeof(uint32_t) * kTicketSlots) return TPL_EWORKSPACE;
    return cuda_rc(cudaMemsetAsync(ws, 0, sizeof(uint32_t) * kTicketSlots, static_cast<cudaStream_t>(stream)));
}

int tpl_pack_layer(const tpl_plan *p, const tpl_layer_weights *w, void *packed, size_t packed_bytes,
                   tpl_stream stream) {
    if (!p || !w || !packed || !al16(packed)) return TPL_EINVAL;
    if ((int64_t)packed_bytes < p->packed_bytes) return TPL_ENOMEM;
    if (!w->wg || !w->wu || !w->wd) return TPL_EINVAL;
    const bool attn = w->wq && w->wk && w->wv && w->wo;
    if (!attn && (w->wq || w->wk || w->wv || w->wo)) return TPL_EINVAL;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const tpl_dims &d = p->d;
    const int64_t es = p->esize, H = d.hidden, hd = d.head_dim, F = d.ffn;
    const int64_t Ks = (int64_t)p->nq_s * hd;
    char *P = static_cast<char *>(packed);
    const char *wq = static_cast<const char *>(w->wq), *wk = static_cast<const char *>(w->wk);
    const char *wv = static_cast<const char *>(w->wv), *wo = static_cast<const char *>(w->wo);
    const char *wg = static_cast<const char *>(w->wg), *wu = static_cast<const char *>(w->wu);
    const char *wd = static_cast<const char *>(w->wd);
    cudaError_t e = cudaSuccess;
    auto ok = [&](cudaError_t r) {
        if (e == cudaSuccess) e = r;
    };
    // padding columns must read as zero
    ok(cudaMemsetAsync(P, 0, (size_t)p->off_g1, st));
    const int64_t lh = (int64_t)p->ld_h * es, lo = (int64_t)p->ld_o * es, lf = (int64_t)p->ld_f * es;
    for (int s = 0; s < p->t; ++s) {
        if (attn) {
            char *dq = P + p->off_qkv + s * p->blk_qkv;
            const int64_t qr = (int64_t)p->nq_s * hd, kr = (int64_t)p->nkv_s * hd;  // rows
            ok(cudaMemcpy2DAsync(dq, lh, wq + s * qr * H * es, H * es, H * es, qr, cudaMemcpyDeviceToDevice, st));
            ok(cudaMemcpy2DAsync(dq + qr * lh, lh, wk + s * kr * H * es, H * es, H * es, kr, cudaMemcpyDeviceToDevice,
                                 st));
            ok(cudaMemcpy2DAsync(dq + (qr + kr) * lh, lh, wv + s * kr * H * es, H * es, H * es, kr,
                                 cudaMemcpyDeviceToDevice, st));
            ok(cudaMemcpy2DAsync(P + p->off_o + s * p->blk_o, lo, wo + s * Ks * es, (int64_t)d.n_q_heads * hd * es,
                                 Ks * es, H, cudaMemcpyDeviceToDevice, st));
        }
        char *dgu = P + p->off_gu + s * p->blk_gu;
        ok(cudaMemcpy2DAsync(dgu, 2 * lh, wg + (int64_t)s * p->F_s * H * es, H * es, H * es, p->F_s,
                             cudaMemcpyDeviceToDevice, st));
        ok(cudaMemcpy2DAsync(dgu + lh, 2 * lh, wu + (int64_t)s * p->F_s * H * es, H * es, H * es, p->F_s,
                             cudaMemcpyDeviceToDevice, st));
        ok(cudaMemcpy2DAsync(P + p->off_d + s * p->blk_d, lf, wd + (int64_t)s * p->F_s * es, F * es,
                             (int64_t)p->F_s * es, H, cudaMemcpyDeviceToDevice, st));
    }
    float *g1 = reinterpret_cast<float *>(P + p->off_g1), *g2 = reinterpret_cast<float *>(P + p->off_g2);
    if (w->gamma_attn) ok(cudaMemcpyAsync(g1, w->gamma_attn, H * 4, cudaMemcpyDeviceToDevice, st));
    else {
        fill_f32_kernel<<<(int)((H + 255) / 256), 256, 0, st>>>(g1, H, 1.0f);
        ok(cudaGetLastError());
    }
    if (w->gamma_mlp) ok(cudaMemcpyAsync(g2, w->gamma_mlp, H * 4, cudaMemcpyDeviceToDevice, st));
    else {
        fill_f32_kernel<<<(int)((H + 255) / 256), 256, 0, st>>>(g2, H, 1.0f);
        ok(cudaGetLastError());
    }
    return cuda_rc(e);
}

int tpl_pack_kv(const tpl_plan *p, const void *unsharded, void *sharded, int32_t batch_cap, int64_t seq_cap,
                tpl_stream stream) {
    if (!p || !unsharded || !sharded || batch_cap < 0 || seq_cap < 0) return TPL_EINVAL;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int64_t row = seq_cap * p->d.head_dim * 2;  // one head's cache bytes
    cudaError_t e = cudaSuccess;
    for (int s = 0; s < p->t && e == cudaSuccess; ++s) {
        const char *src = static_cast<const char *>(unsharded) + (int64_t)s * p->nkv_s * row;
        char *dst = static_cast<char *>(sharded) + (int64_t)s * batch_cap * p->nkv_s * row;
        e = cudaMemcpy2DAsync(dst, p->nkv_s * row, src, (int64_t)p->d.n_kv_heads * row, p->nkv_s * row, batch_cap,
                              cudaMemcpyDeviceToDevice, st);
    }
    return cuda_rc(e);
}

int tpl_qkv(tpl_plan *p, const void *packed, const tpl_kv *kv, const void *x, int32_t B, int64_t S, float *q,
            float *k_new, float *v_new, void *ws, size_t ws_bytes, tpl_stream stream) {
    if (B == 0) return TPL_OK;
    Ctx c;
    int rc = make_ctx(p, ws, ws_bytes, B, S, stream, &c);
    if (rc != TPL_OK) return rc;
    if (!packed || !x || !q || !al16(x) || !al16(packed)) return TPL_EINVAL;
    if ((rc = check_kv(kv, B, S)) != TPL_OK) return rc;
    if ((k_new && !al16(k_new)) || (v_new && !al16(v_new)) || (!k_new != !v_new)) return TPL_EINVAL;
    return run_qkv(c, static_cast<const char *>(packed), kv, x, q, k_new, v_new);
}

int tpl_attn_decode(tpl_plan *p, const tpl_kv *kv, const float *q, const float *k_new, const float *v_new, int32_t B,
                    int64_t S, void *o, void *ws, size_t ws_bytes, tpl_stream stream) {
    if (B == 0) return TPL_OK;
    Ctx c;
    int rc = make_ctx(p, ws, ws_bytes, B, S, stream, &c);
    if (rc != TPL_OK) return rc;
    if (!q || !o || !al16(q) || (!k_new != !v_new)) return TPL_EINVAL;
    if ((rc = check_kv(kv, B, S)) != TPL_OK) return rc;
    return run_attn(c, kv, q, k_new, v_new, o);
}

int tpl_o_proj(tpl_plan *p, const void *packed, const void *o, const void *x, int32_t B, float *h, float *partials,
               void *ws, size_t ws_bytes, tpl_stream stream) {
    if (B == 0) return TPL_OK;
    Ctx c;
    int rc = make_ctx(p, ws, ws_bytes, B, 0, stream, &c);
    if (rc != TPL_OK) return rc;
    if (!packed || !o || !al16(o) || (!partials && !h)) return TPL_EINVAL;
    const bool resid = (p->d.flags & TPL_RESIDUAL) != 0;
    if (resid && !partials && !x) return TPL_EINVAL;
    return run_o(c, static_cast<const char *>(packed), o, resid ? x : nullptr, h, partials);
}

int tpl_gate_up(tpl_plan *p, const void *packed, const void *h, int32_t h_is_act, int32_t B, void *act, void *ws,
                size_t ws_bytes, tpl_stream stream) {
    if (B == 0) return TPL_OK;
    Ctx c;
    int rc = make_ctx(p, ws, ws_bytes, B, 0, stream, &c);
    if (rc != TPL_OK) return rc;
    if (!packed || !h || !act || !al16(h)) return TPL_EINVAL;
    return run_gu(c, static_cast<const char *>(packed), h, h_is_act ? 1 : 0, act);
}

int tpl_down_proj(tpl_plan *p, const void *packed, const void *act, const float *h, int32_t B, void *y, float *y32,
                  float *partials, void *ws, size_t ws_bytes, tpl_stream stream) {
    if (B == 0) return TPL_OK;
    Ctx c;
    int rc = make_ctx(p, ws, ws_bytes, B, 0, stream, &c);
    if (rc != TPL_OK) return rc;
    if (!packed || !act || !al16(act) || (!partials && !y && !y32)) return TPL_EINVAL;
    const bool resid = (p->d.flags & TPL_RESIDUAL) != 0;
    if (resid && !partials && !h) return TPL_EINVAL;
    return run_down(c, static_cast<const char *>(packed), act, resid ? h : nullptr, 1, y, y32, partials);
}

int tpl_reduce_partials(tpl_plan *p, const float *P, const void *resid, int32_t resid_is_f32, int32_t B, float *out32,
                        void *out_act, tpl_stream stream) {
    if (!p || !P || B < 0 || (!out32 && !out_act)) return TPL_EINVAL;
    if (B == 0) return TPL_OK;
    return run_reduce(p, static_cast<cudaStream_t>(stream), P, resid, resid_is_f32 ? 1 : 0, B, out32, out_act);
}

int tpl_mlp_block(tpl_plan *p, const void *packed, const void *x, int32_t B, void *y, float *y32, void *ws,
                  size_t ws_bytes, int32_t reduce_mode, tpl_stream stream) {
    if (B == 0) return TPL_OK;
    if (reduce_mode != TPL_REDUCE_FUSED && reduce_mode != TPL_REDUCE_SEPARATE) return TPL_EINVAL;
    Ctx c;
    int rc = make_ctx(p, ws, ws_bytes, B, 0, stream, &c);
    if (rc != TPL_OK) return rc;
    if (!packed || !x || !al16(x) || (!y && !y32)) return TPL_EINVAL;
    const char *pk = static_cast<const char *>(packed);
    const bool resid = (p->d.flags & TPL_RESIDUAL) != 0;
    void *act = c.ws + c.L.act;
    float *P = reinterpret_cast<float *>(c.ws + c.L.P);
    rc = run_gu(c, pk, x, 1, act);
    if (rc != TPL_OK) return rc;
    if (reduce_mode == TPL_REDUCE_FUSED) return run_down(c, pk, act, resid ? x : nullptr, p->f32, y, y32, nullptr);
    rc = run_down(c, pk, act, nullptr, 0, nullptr, nullptr, P);
    if (rc != TPL_OK) return rc;
    return run_reduce(p, c.st, P, resid ? x : nullptr, p->f32, B, y32, y);
}

int tpl_decode_layer(tpl_plan *p, const void *packed, const tpl_kv *kv, const void *x, int32_t B, int64_t S, void *y,
                     float *y32, void *ws, size_t ws_bytes, int32_t reduce_mode, tpl_stream stream) {
    if (B == 0) return TPL_OK;
    if (reduce_mode != TPL_REDUCE_FUSED && reduce_mode != TPL_REDUCE_SEPARATE) return TPL_EINVAL;
    Ctx c;
    int rc = make_ctx(p, ws, ws_bytes, B, S, stream, &c);
    if (rc != TPL_OK) return rc;
    if (!packed || !x || !al16(x) || !al16(packed) || (!y && !y32)) return TPL_EINVAL;
    if ((rc = check_kv(kv, B, S)) != TPL_OK) return rc;
    return decode_layer(c, static_cast<const char *>(packed), kv, x, y, y32, reduce_mode);
}

int tpl_decode_stack(tpl_plan *p, const void *const *packed_per_layer, const tpl_kv *kv_per_layer, const void *x,
                     int32_t B, int64_t S, void *y, float *y32, void *ws, size_t ws_bytes, int32_t reduce_mode,
                     tpl_stream stream) {
    if (B == 0) return TPL_OK;
    if (reduce_mode != TPL_REDUCE_FUSED && reduce_mode != TPL_REDUCE_SEPARATE) return TPL_EINVAL;
    Ctx c;
    int rc = make_ctx(p, ws, ws_bytes, B, S, stream, &c);
    if (rc != TPL_OK) return rc;
    if (!packed_per_layer || !kv_per_layer || !x || !al16(x) || (!y && !y32)) return TPL_EINVAL;
    const int L = p->d.n_layers;
    for (int l = 0; l < L; ++l) {
        if (!packed_per_layer[l] || !al16(packed_per_layer[l])) return TPL_EINVAL;
        if ((rc = check_kv(&kv_per_layer[l], B, S)) != TPL_OK) return rc;
    }
    void *buf[2] = {c.ws + c.L.ybuf0, c.ws + c.L.ybuf1};
    const void *cur = x;
    for (int l = 0; l < L; ++l) {
        const bool last = l == L - 1;
        // the down projection of a layer followed by another writes that
        // layer's QKV operand
        c.has_next = !last;
        c.next_gamma = last ? nullptr
                            : reinterpret_cast<const float *>(static_cast<const char *>(packed_per_layer[l + 1]) +
                                                              p->off_g1);
        void *out = last ? y : buf[l & 1];
        float *out32 = last ? y32 : nullptr;
        if (last && !y) out = buf[l & 1];
        rc = decode_layer(c, static_cast<const char *>(packed_per_layer[l]), &kv_per_layer[l], cur, out, out32,
                          reduce_mode);
        if (rc != TPL_OK) return rc;
        cur = out;
    }
    return TPL_OK;
}

int tpl_prefill_layer(tpl_plan *p, const void *packed, const tpl_kv *kv, const void *x, int32_t T, void *y,
                      float *y32, void *ws, size_t ws_bytes, int32_t reduce_mode, tpl_stream stream) {
    return tpl_prefill_chunk(p, packed, kv, x, T, 0, y, y32, ws, ws_bytes, reduce_mode, stream);
}

int tpl_prefill_chunk(tpl_plan *p, const void *packed, const tpl_kv *kv, const void *x, int32_t T, int64_t start,
                      void *y, float *y32, void *ws, size_t ws_bytes, int32_t reduce_mode, tpl_stream stream) {
    if (!p || T < 0 || start < 0) return TPL_EINVAL;
    if (reduce_mode != TPL_REDUCE_FUSED && reduce_mode != TPL_REDUCE_SEPARATE) return TPL_EINVAL;
    if (T == 0) return TPL_OK;
    if (p->f32) return TPL_EUNSUPPORTED;
    if (!packed || !x || !ws || !al16(packed) || !al16(x) || !al16(ws) || (!y && !y32)) return TPL_EINVAL;
    if ((y && !al16(y)) || (y32 && !al16(y32))) return TPL_EINVAL;
    int rc = check_kv(kv, 1, start + T - 1);
    if (rc != TPL_OK) return rc;
    if (start + T > 0x7fffffffll) return TPL_EUNSUPPORTED;  // key positions are 32-bit in the kernels
    PrefillWs L;
    if ((rc = prefill_ws_layout(p, T, &L)) != TPL_OK) return rc;
    if (ws_bytes < L.total) return TPL_EWORKSPACE;
    return prefill_layer(p, static_cast<const char *>(packed), kv, x, T, (int)start, y, y32, static_cast<char *>(ws),
                         L, reduce_mode, static_cast<cudaStream_t>(stream));
}

int tpl_decode_kernel_count(const tpl_plan *p, int32_t B, int32_t reduce_mode, int32_t n_layers, int32_t *count) {
    if (!p || !count || B < 1 || n_layers < 1) return TPL_EINVAL;
    if (reduce_mode != TPL_REDUCE_FUSED && reduce_mode != TPL_REDUCE_SEPARATE) return TPL_EINVAL;
    if (B > (p->f32 ? kMaxBatchCuda : kMaxBatch)) return TPL_EUNSUPPORTED;
    const bool sep = reduce_mode == TPL_REDUCE_SEPARATE;
    int64_t n;
    if (use_tc(p, OP_QKV, B)) {
        // QKV, attention, O, gate/up, down; the operand kernel before QKV and
        // gate/up unless the fused O and the previous layer's down wrote it
        n = sep ? 9ll * n_layers : 5ll * n_layers + 1;
    } else {
        n = (sep ? 7ll : 5ll) * n_layers;
    }
    if (p->rope) n += n_layers;
    if (n > 0x7fffffff) return TPL_EINVAL;
    *count = (int32_t)n;
    return TPL_OK;
}

int tpl_trace_read(void *records, int32_t max_records, int32_t *n_records) {
#ifdef TPL_TRACE
    if (!n_records || max_records < 0 || (max_records > 0 && !records)) return TPL_EINVAL;
    if (cudaDeviceSynchronize() != cudaSuccess) return TPL_ECUDA;
    unsigned n = 0;
    if (cudaMemcpyFromSymbol(&n, g_trace_n, sizeof(n)) != cudaSuccess) return TPL_ECUDA;
    if (n > kTraceMax) n = kTraceMax;
    const unsigned take = n < (unsigned)max_records ? n : (unsigned)max_records;
    if (take && cudaMemcpyFromSymbol(records, g_trace, take * sizeof(TraceRec)) != cudaSuccess) return TPL_ECUDA;
    const unsigned z = 0;
    if (cudaMemcpyToSymbol(g_trace_n, &z, sizeof(z)) != cudaSuccess) return TPL_ECUDA;
    *n_records = (int32_t)take;
    return TPL_OK;
#else
    (void)records;
    (void)max_records;
    if (n_records) *n_records = 0;
    return TPL_EUNSUPPORTED;
#endif
}

int tpl_last_device_error(const tpl_plan *p, tpl_stream stream) {
    (void)p;
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return TPL_ECUDA;
    unsigned v = 0;
    if (cudaMemcpyFromSymbol(&v, g_err_word, sizeof(v)) != cudaSuccess) return TPL_ECUDA;
    if (v) {
        const unsigned z = 0;
        if (cudaMemcpyToSymbol(g_err_word, &z, sizeof(z)) != cudaSuccess) return TPL_ECUDA;
        return TPL_EDEVICE;
    }
    return TPL_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free variant of tpl_attn_decode.  For callers that cannot
// allocate device memory (a plugin whose host application owns the device
// budget, a serving loop that must stay out of the allocator): the split
// partials and arrival counters live in this fixed array of static device
// memory instead of a caller-provided workspace.  Every device that loads the
// library holds the array until the process exits.  Calls share it and it
// keeps the previous call's contents, so each call clears the counters it
// uses first; calls that overlap on the GPU race on it.
// ---------------------------------------------------------------------------
static __device__ __align__(256) unsigned char g_attn_scratch[TPL_ATTN_STATIC_SCRATCH_BYTES];

namespace {
std::atomic<void *> g_attn_scratch_addr[64];  // device address of g_attn_scratch, per device

size_t round256(size_t v) { return (v + 255) / 256 * 256; }
}  // namespace

extern "C" int tpl_attn_decode_static(tpl_plan *p, const tpl_kv *kv, const float *q, const float *k_new,
                                      const float *v_new, int32_t B, int64_t S, void *o, tpl_stream stream) {
    if (!p || !q || !o || !al16(q) || B < 0 || S < 0 || (!k_new != !v_new)) return TPL_EINVAL;
    if (B == 0) return TPL_OK;
    if (B > kMaxBatch) return TPL_EUNSUPPORTED;
    int rc = check_kv(kv, B, S);
    if (rc != TPL_OK) return rc;
    const int64_t keys = k_new ? S : S + 1;
    // the same kernel and split geometry tpl_attn_decode chooses, so the two
    // calls give identical bits
    AttnGeom g;
    int kind = 0;
    if ((rc = attn_select(p, B, keys, &g, &kind)) != TPL_OK) return rc;
    const size_t off_ml = round256((size_t)g.pairs * sizeof(unsigned));
    const size_t cpp = (size_t)attn_cpp(g, kind);  // partials are per CTA
    const size_t off_o = off_ml + round256((size_t)g.pairs * cpp * p->g * 2 * sizeof(float));
    const size_t need = off_o + round256((size_t)g.pairs * cpp * p->g * p->d.head_dim * sizeof(float));
    if (need > TPL_ATTN_STATIC_SCRATCH_BYTES) return TPL_ENOMEM;
    // Set-up, once per device with that device current: the array's device
    // address (in host code its name is only a host-side stand-in).
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return TPL_ECUDA;
    void *base = g_attn_scratch_addr[dev].load();
    if (!base) {
        if (cudaGetSymbolAddress(&base, g_attn_scratch) != cudaSuccess || !base) return TPL_ECUDA;
        g_attn_scratch_addr[dev].store(base);
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    char *scratch = static_cast<char *>(base);
    // The arrival counters must start at zero.
    if (cudaMemsetAsync(scratch, 0, (size_t)g.pairs * sizeof(unsigned), st) != cudaSuccess) return TPL_ECUDA;
    return attn_launch(p, kv, q, k_new, v_new, B, keys, o, g, kind, reinterpret_cast<unsigned *>(scratch),
                       reinterpret_cast<float *>(scratch + off_ml), reinterpret_cast<float *>(scratch + off_o), st);
}
