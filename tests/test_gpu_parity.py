"""GPU parity: the CUDA path through the C-ABI against the oracle, element by
element on the same seeded inputs.  Tolerance for bf16-in / fp32-accumulate
outputs: |gpu - oracle| <= 2e-2 * (|oracle| + RMS(oracle)); fused and separate
reductions bitwise equal; cross-t agreement 1e-3 in the fp32 mode."""
import numpy as np
import pytest
import torch

from tests.conftest import has_gpu

pytestmark = pytest.mark.gpu

if has_gpu():
    import oracle
    from megatron_tensor_transformer_plan_b200 import synth, tpl
    from tests.gpu_util import (assert_close_rel, make_layer, new_kv_slot, oracle_decode, oracle_dims,
                                oracle_weights, run_steps, to_np)


def _check_layer(L, ref_y, tr, mode_both=True):
    steps = run_steps(L, tpl.TPL_REDUCE_FUSED)
    d = L.dims
    assert_close_rel(to_np(steps["q"]).reshape(L.B, -1), tr["q"], what="q")
    kk, vv = new_kv_slot(L)
    assert_close_rel(to_np(kk), tr["k_new"], what="k_new (cache slot S)")
    assert_close_rel(to_np(vv), tr["v_new"], what="v_new (cache slot S)")
    assert_close_rel(to_np(steps["k_new"]).reshape(L.B, -1), tr["k_new"], what="k_new fp32")
    assert_close_rel(to_np(steps["v_new"]).reshape(L.B, -1), tr["v_new"], what="v_new fp32")
    # the cache holds the bf16 rounding of the fp32 values
    assert torch.equal(kk, steps["k_new"].reshape(L.B, -1).bfloat16())
    assert_close_rel(to_np(steps["attn"]), tr["attn"], what="attention output")
    assert_close_rel(to_np(steps["h"]), tr["h"], what="h")
    assert_close_rel(to_np(steps["act"]), tr["act"], what="act")
    assert_close_rel(to_np(steps["y32"]), ref_y, what="y32")
    assert_close_rel(to_np(steps["y"]), ref_y, what="y")
    # the one-call layer runs the same kernels: identical bits
    y = torch.empty_like(steps["y"])
    y32 = torch.empty_like(steps["y32"])
    L.plan.decode_layer(L.packed, L.kv, L.x, L.S, y, y32, L.ws, tpl.TPL_REDUCE_FUSED)
    torch.cuda.synchronize()
    assert torch.equal(y, steps["y"]) and torch.equal(y32, steps["y32"])
    if mode_both:
        ys = torch.empty_like(y)
        ys32 = torch.empty_like(y32)
        L.plan.decode_layer(L.packed, L.kv, L.x, L.S, ys, ys32, L.ws, tpl.TPL_REDUCE_SEPARATE)
        torch.cuda.synchronize()
        assert torch.equal(ys32, y32), "fused and separate reductions differ"
        assert torch.equal(ys, y)
    assert L.plan.last_device_error() == tpl.TPL_OK
    return steps


SMALL = [
    # H, nq, nkv, F, t, B, S, gamma_std
    (512, 8, 2, 1376, 2, 3, 37, 0.0),       # ragged batch, short cache
    (256, 4, 4, 704, 4, 1, 0, 0.0),         # MHA (g = 1), S = 0: one key
    (1024, 16, 8, 2816, 8, 16, 300, 0.02),  # B = 16, t = 8, non-unit gains
    (768, 12, 4, 1056, 4, 5, 129, 0.0),     # F/t = 264 (ragged 128-column block), g = 3
    (512, 16, 1, 512, 1, 2, 1000, 0.0),     # g = 16
]


@pytest.mark.parametrize("case", SMALL)
def test_decode_layer_small(gpu, case):
    H, nq, nkv, F, t, B, S, gs = case
    L = make_layer(H, nq, nkv, 128, F, t, B, S, gamma_std=gs, S_cap=S + 3)
    ref_y, tr = oracle_decode(L)
    _check_layer(L, ref_y, tr)


def test_empty_cache_attention_is_new_value(gpu):
    """S = 0: one key, weight exactly 1, so the attention output is v_new
    (exactly, up to the output's bf16 rounding)."""
    L = make_layer(1024, 16, 4, 128, 2816, 4, 3, 0)
    st = run_steps(L)
    g = 16 // 4
    v = st["v_new"]  # [B][n_kv][d]
    expect = v.repeat_interleave(g, dim=1).reshape(L.B, -1).bfloat16()
    assert torch.equal(st["attn"], expect)


def test_kv_cache_only_slot_s_changes(gpu):
    L = make_layer(512, 8, 2, 128, 1376, 2, 3, 37, S_cap=45)
    before_k, before_v = L.k.clone(), L.v.clone()
    run_steps(L)
    t, B, nkv_s = 2, 3, 1
    vk = L.k.view(t, B, nkv_s, 45, 128)
    bk = before_k.view(t, B, nkv_s, 45, 128)
    mask = torch.ones(45, dtype=torch.bool, device=L.k.device)
    mask[37] = False
    assert torch.equal(vk[:, :, :, mask], bk[:, :, :, mask])
    assert torch.equal(L.v.view(t, B, nkv_s, 45, 128)[:, :, :, mask], before_v.view(t, B, nkv_s, 45, 128)[:, :, :, mask])


def test_config1_tiny_mlp_block(gpu):
    """Hidden 256, ffn 688 (344 per shard), t = 2, one token, no norm, no
    residual: y = sum_s (silu(x Wg_s^T) * (x Wu_s^T)) Wd_s^T."""
    H, F, t = 256, 688, 2
    L = make_layer(H, 2, 2, 128, F, t, 1, 0, flags=0, mlp_only=True)
    w = oracle_weights(L)
    od = oracle_dims(L)
    x = to_np(L.x)
    ref, parts = oracle.mlp_sharded(od, w, t, x, partials=True)
    ref1 = oracle.mlp_sharded(od, w, 1, x)
    np.testing.assert_allclose(ref, ref1, rtol=1e-12, atol=1e-12 * np.abs(ref1).max())
    y = torch.empty((1, H), dtype=torch.bfloat16, device=gpu)
    y32 = torch.empty((1, H), dtype=torch.float32, device=gpu)
    L.plan.mlp_block(L.packed, L.x, y, y32, L.ws, tpl.TPL_REDUCE_FUSED)
    ys = torch.empty_like(y)
    ys32 = torch.empty_like(y32)
    L.plan.mlp_block(L.packed, L.x, ys, ys32, L.ws, tpl.TPL_REDUCE_SEPARATE)
    # shard partials of the row-split down projection
    act = torch.empty((1, F), dtype=torch.bfloat16, device=gpu)
    L.plan.gate_up(L.packed, L.x, act, L.ws, h_is_act=True)
    P = torch.empty((t, 1, H), dtype=torch.float32, device=gpu)
    L.plan.down_proj(L.packed, act, None, partials=P, ws=L.ws)
    torch.cuda.synchronize()
    assert_close_rel(to_np(y32), ref, what="y32")
    assert_close_rel(to_np(y), ref, what="y")
    assert torch.equal(y32, ys32) and torch.equal(y, ys)
    for s in range(t):
        assert_close_rel(to_np(P[s]), parts[s], what=f"partial {s}")
    # the partials add (in shard order) to the fused result exactly
    acc = P[0].clone()
    for s in range(1, t):
        acc = acc + P[s]
    assert torch.equal(acc, y32)


@pytest.mark.parametrize("t", [1, 2, 4])
@pytest.mark.parametrize("B", [1, 16])
def test_config2_7b_layer(gpu, t, B):
    """7B-shaped layer: hidden 4096, 32/32 heads, ffn 11008, KV length 2048."""
    L = make_layer(4096, 32, 32, 128, 11008, t, B, 2048, seed=0)
    ref_y, tr = oracle_decode(L)
    _check_layer(L, ref_y, tr, mode_both=(B == 16))


@pytest.mark.slow
@pytest.mark.parametrize("gemv_mode", [4, 0])
def test_config3_70b_layer(gpu, gemv_mode):
    """70B-shaped layer, t = 4 (2 kv heads per shard), batch 16, KV length 8192;
    the default kernel choice (4) and the mma.sync projections (0)."""
    L = make_layer(8192, 64, 8, 128, 28672, 4, 16, 8192, seed=0)
    L.plan.set_option(tpl.TPL_OPT_GEMV_MODE, gemv_mode)
    ref_y, tr = oracle_decode(L)
    _check_layer(L, ref_y, tr)


@pytest.mark.slow
@pytest.mark.parametrize("gemv_mode", [4, 0])
def test_stack_shape_layer(gpu, gemv_mode):
    """One layer at the 80-layer stack's shape: t = 8, batch 4, KV length 4096."""
    L = make_layer(8192, 64, 8, 128, 28672, 8, 4, 4096, seed=0, layer=39)
    L.plan.set_option(tpl.TPL_OPT_GEMV_MODE, gemv_mode)
    ref_y, tr = oracle_decode(L)
    _check_layer(L, ref_y, tr)


def test_cross_t_fp32_mode(gpu):
    """fp32 weights/activations: the t = 2, 4, 8 layouts agree with t = 1 to
    1e-3 (only the association of the shard sums differs)."""
    H, nq, nkv, F, B, S = 1024, 16, 8, 2048, 4, 100
    flags = tpl.TPL_NORM | tpl.TPL_RESIDUAL | tpl.TPL_FP32_WEIGHTS
    outs = {}
    for t in (1, 2, 4, 8):
        L = make_layer(H, nq, nkv, 128, F, t, B, S, flags=flags, seed=3)
        y = torch.empty((B, H), dtype=torch.float32, device=gpu)
        L.plan.decode_layer(L.packed, L.kv, L.x, S, y, None, L.ws, tpl.TPL_REDUCE_FUSED)
        torch.cuda.synchronize()
        outs[t] = to_np(y)
        if t == 1:
            ref_y, _ = oracle_decode(L)
            assert_close_rel(outs[1], ref_y, what="fp32 mode vs oracle")
    for t in (2, 4, 8):
        assert_close_rel(outs[t], outs[1], tol=1e-3, what=f"t={t} vs t=1")


def test_gemv_ffma_mode_matches(gpu):
    L = make_layer(1024, 16, 8, 128, 2816, 4, 4, 64)
    ref_y, tr = oracle_decode(L)
    L.plan.set_option(tpl.TPL_OPT_GEMV_MODE, 2)
    steps = run_steps(L)
    assert_close_rel(to_np(steps["y"]), ref_y, what="y (FFMA mode)")
    assert_close_rel(to_np(steps["act"]), tr["act"], what="act (FFMA mode)")


def test_stack_equals_layer_sequence(gpu):
    """The stack call is the layer call applied L times (same bits), and it
    counts 2L reduction points."""
    H, nq, nkv, F, t, B, S, NL = 512, 8, 4, 1024, 4, 2, 50, 4
    layers = [make_layer(H, nq, nkv, 128, F, t, B, S, seed=5, layer=l, n_layers=NL) for l in range(NL)]
    plan = layers[0].plan
    x = layers[0].x
    ws = plan.workspace(B, S)
    # the stack writes slot S of every layer's cache; snapshot to rerun
    snaps = [(L.k.clone(), L.v.clone()) for L in layers]
    y_stack = torch.empty_like(x)
    plan.reset_counters()
    plan.decode_stack([L.packed for L in layers], [L.kv for L in layers], x, S, y_stack, None, ws)
    torch.cuda.synchronize()
    assert plan.reduction_count() == 2 * NL
    for L, (k, v) in zip(layers, snaps):
        L.k.copy_(k)
        L.v.copy_(v)
    cur = x
    for L in layers:
        nxt = torch.empty_like(x)
        plan.decode_layer(L.packed, L.kv, cur, S, nxt, None, ws)
        cur = nxt
    torch.cuda.synchronize()
    assert torch.equal(cur, y_stack)
    assert plan.reduction_count() == 4 * NL
    plan.reset_counters()
    ys = torch.empty_like(x)
    plan.decode_stack([L.packed for L in layers], [L.kv for L in layers], x, S, ys, None, ws,
                      tpl.TPL_REDUCE_SEPARATE)
    torch.cuda.synchronize()
    assert plan.reduction_count() == 2 * NL
    assert torch.equal(ys, y_stack)


def test_repeated_calls_are_deterministic(gpu):
    L = make_layer(1024, 16, 8, 128, 2816, 8, 16, 500)
    a = run_steps(L)["y32"].clone()
    for _ in range(3):
        b = run_steps(L)["y32"]
        assert torch.equal(a, b)


@pytest.mark.parametrize("case", [(1024, 16, 8, 2816, 8, 4, 700), (512, 8, 2, 1376, 2, 3, 37),
                                  (256, 4, 4, 704, 4, 1, 0)])
def test_decode_attention_kernels_agree(gpu, case):
    """The staged attention kernel (default), the register-streamed one
    (TPL_OPT_DECODE_ATTN 1) and the TMA-streamed one (2): each against the
    oracle, and close to each other."""
    H, nq, nkv, F, t, B, S = case
    outs = []
    for mode in (0, 1, 2):
        L = make_layer(H, nq, nkv, 128, F, t, B, S, S_cap=S + 3)
        L.plan.set_option(tpl.TPL_OPT_DECODE_ATTN, mode)
        ref_y, tr = oracle_decode(L)
        st = run_steps(L)
        assert_close_rel(to_np(st["attn"]), tr["attn"], what=f"attention (mode {mode})")
        assert_close_rel(to_np(st["y"]), ref_y, what=f"y (mode {mode})")
        outs.append(to_np(st["attn"]))
    assert_close_rel(outs[0], outs[1], tol=8e-3, what="staged vs register attention")
    assert_close_rel(outs[0], outs[2], tol=8e-3, what="staged vs TMA-streamed attention")


TMA_ATTN_CASES = [
    # H, nq, nkv, F, t, B, S, S_cap extra: blocks of 64 keys laid end to end over every SM
    (1024, 16, 8, 2816, 8, 4, 4096, 1),    # the stack's attention shape at small hidden: 32 pairs
    (1024, 16, 8, 2816, 4, 16, 1000, 5),   # 128 pairs, ragged last block, several pairs per CTA
    (512, 8, 8, 1024, 2, 3, 1, 1),         # one cached key (a block of one valid row), g = 1
    (512, 8, 2, 1376, 2, 2, 63, 2),        # 63 keys: one block short of a full one
    (512, 8, 2, 1376, 2, 2, 65, 1),        # 65 keys: a full block and a block of one key
    (768, 12, 4, 1056, 4, 5, 129, 9),      # g = 3
    (1024, 8, 1, 1024, 1, 2, 5000, 3),     # one kv head per sequence: a pair spans many CTAs
    (2048, 32, 32, 2048, 1, 20, 300, 1),   # 640 pairs: many pairs per CTA
]


@pytest.mark.parametrize("case", TMA_ATTN_CASES)
def test_tma_attention_kernel(gpu, case):
    """The TMA-streamed decode attention (TPL_OPT_DECODE_ATTN 2) at ragged
    cache lengths and pair counts from one CTA per many pairs to many CTAs per
    pair, against the oracle, with the new token given separately and read
    from cache slot S."""
    H, nq, nkv, F, t, B, S, extra = case
    L = make_layer(H, nq, nkv, 128, F, t, B, S, S_cap=S + extra, seed=17)
    L.plan.set_option(tpl.TPL_OPT_DECODE_ATTN, 2)
    ref_y, tr = oracle_decode(L)
    st = run_steps(L)
    assert_close_rel(to_np(st["attn"]), tr["attn"], what="attention (new token separate)")
    assert_close_rel(to_np(st["y"]), ref_y, what="y")
    # the new token read from cache slot S (written by the QKV step above, bf16):
    # against the register-streamed kernel reading the same cache
    o2 = torch.empty_like(st["attn"])
    L.plan.attn_decode(L.kv, st["q"], S, o2, L.ws)
    L.plan.set_option(tpl.TPL_OPT_DECODE_ATTN, 1)
    o1 = torch.empty_like(st["attn"])
    L.plan.attn_decode(L.kv, st["q"], S, o1, L.ws)
    torch.cuda.synchronize()
    assert_close_rel(to_np(o2), to_np(o1), tol=8e-3, what="attention (new token from the cache)")
    assert L.plan.last_device_error() == tpl.TPL_OK
