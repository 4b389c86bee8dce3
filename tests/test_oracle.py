"""Pins for the oracle: what the pages and the mathematics fix, independent of
the oracle's own code.  CPU only.

Each test is chosen so that a plausible mistake in the oracle (a dropped term,
a wrong sign, a transposed operand, a wrong head mapping, a wrong softmax
scale, a wrong summation) fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle
from tests import np_reference

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


def rng(seed=0):
    return np.random.default_rng(seed)


def rand_bf16_bits(r, shape, std):
    """Random values rounded to bf16 (truncation of float32 bits is fine for a
    test input: the result is some bf16 value), returned as raw bits."""
    a = (r.standard_normal(shape) * std).astype(np.float32)
    return (a.view(np.uint32) >> 16).astype(np.uint16)


def small_layer(r, H=32, nq=4, nkv=2, d=8, F=48, std=0.2, bf16=True):
    shapes = {"wq": (nq * d, H), "wk": (nkv * d, H), "wv": (nkv * d, H), "wo": (H, nq * d),
              "wg": (F, H), "wu": (F, H), "wd": (H, F)}
    if bf16:
        w = {k: rand_bf16_bits(r, s, std) for k, s in shapes.items()}
    else:
        w = {k: f32(r.standard_normal(s) * std) for k, s in shapes.items()}
    w["gamma_attn"] = f32(1 + 0.1 * r.standard_normal(H))
    w["gamma_mlp"] = f32(1 + 0.1 * r.standard_normal(H))
    return w


# --------------------------------------------------------------------------
# The pages' worked numbers
# --------------------------------------------------------------------------

def test_kv_formula_worked_example():
    g = golden("kv_footprint.json")
    per_seq = oracle.kv_bytes_per_shard(g["layers"], g["kv_heads"], g["head_dim"], g["seq"],
                                        g["bytes_per_elem"], 1, 1)
    assert per_seq == g["bytes_per_sequence"]
    assert per_seq // g["bytes_per_elem"] == g["elements_per_sequence"]
    assert oracle.kv_bytes_per_shard(g["layers"], g["kv_heads"], g["head_dim"], g["seq"],
                                     g["bytes_per_elem"], g["batch"], 1) == g["bytes_batch"]
    assert oracle.kv_bytes_per_shard(g["layers"], g["kv_heads"], g["head_dim"], g["seq"],
                                     g["bytes_per_elem"], g["batch"], g["t"]) == g["bytes_per_gpu"]
    # the page's rounded figures are binary gigabytes
    assert g["bytes_per_sequence"] == 2.5 * 2**30
    assert g["bytes_batch"] == 40 * 2**30
    assert g["bytes_per_gpu"] == 10 * 2**30


def test_reductions_per_pass():
    g = golden("reductions.json")
    assert oracle.reductions_per_pass(g["layers"]) == g["per_pass"]
    assert oracle.reductions_per_pass(1) == g["per_layer"]
    assert 8192 * 2 == g["message_bytes_per_token"]


def test_weight_footprint_70b():
    g = golden("weights_footprint.json")
    d = oracle.Dims(8192, 64, 8, 128, 28672)
    per_shard = oracle.layer_params_per_shard(d, g["t"])
    full = oracle.layer_params_per_shard(d, 1)
    assert full == 4 * per_shard  # weights divide exactly by t
    total_gb = 80 * full * 2 / 1e9
    per_gpu_gb = 80 * per_shard * 2 / 1e9
    assert abs(total_gb - g["approx_total_GB"]) / g["approx_total_GB"] < g["rel_tolerance"]
    assert abs(per_gpu_gb - g["approx_per_gpu_GB_t4"]) / g["approx_per_gpu_GB_t4"] < g["rel_tolerance"]
    # hand count of the Llama-3.1-70B-shaped layer: q 8192x8192, k/v 1024x8192,
    # o 8192x8192, gate/up 28672x8192, down 8192x28672
    assert full == 8192 * 8192 * 2 + 1024 * 8192 * 2 + 28672 * 8192 * 3


# --------------------------------------------------------------------------
# Shard maps: the ownership rule and its consequences
# --------------------------------------------------------------------------

@pytest.mark.parametrize("dims", [(8192, 64, 8, 128, 28672), (4096, 32, 32, 128, 11008),
                                  (256, 4, 2, 64, 688)])
@pytest.mark.parametrize("t", [1, 2, 4, 8])
def test_plan_maps_invariants(dims, t):
    d = oracle.Dims(*dims)
    m = oracle.plan_maps(d, t)
    H, nq, nkv, hd, F = dims
    if nq % t or nkv % t or F % t:
        assert m is None
        return
    g = nq // nkv
    # every shard owns the same number of whole heads, contiguously
    for s in range(t):
        owned = np.nonzero(m["q_shard"] == s)[0]
        assert len(owned) == nq // t
        assert np.all(np.diff(owned) == 1)
        assert list(m["q_local"][owned]) == list(range(nq // t))
    # local attention needs no communication: the kv head a query head reads
    # lives on the same shard
    for h in range(nq):
        assert m["kv_shard"][h // g] == m["q_shard"][h]
    assert np.all(np.bincount(m["ffn_shard"], minlength=t) == F // t)
    assert np.all(np.diff(m["ffn_shard"]) >= 0)


@pytest.mark.parametrize("dims", [(8192, 64, 8, 128, 28672), (4096, 32, 32, 128, 11008),
                                  (256, 4, 2, 64, 688), (1024, 16, 8, 128, 2816)])
@pytest.mark.parametrize("t", [1, 2, 4, 8])
def test_plan_maps_rank_order(dims, t):
    """The ownership rule fixes which block each rank holds, not only that the
    blocks are contiguous: rank r holds the r-th block of n/t query heads, of
    kv heads and of ffn columns, in ascending order ("Tensor parallel scaling
    curves", "What tensor parallelism actually splits").  A reversed or
    rotated rank order passes the invariants above but fails here."""
    d = oracle.Dims(*dims)
    m = oracle.plan_maps(d, t)
    H, nq, nkv, hd, F = dims
    if nq % t or nkv % t or F % t:
        assert m is None
        return
    for r in range(t):
        # the block written out from the rule, element by element
        q_block = list(range(r * (nq // t), (r + 1) * (nq // t)))
        kv_block = list(range(r * (nkv // t), (r + 1) * (nkv // t)))
        f_block = list(range(r * (F // t), (r + 1) * (F // t)))
        assert list(np.nonzero(m["q_shard"] == r)[0]) == q_block
        assert list(np.nonzero(m["kv_shard"] == r)[0]) == kv_block
        assert list(np.nonzero(m["ffn_shard"] == r)[0]) == f_block
        assert [int(m["q_local"][h]) for h in q_block] == list(range(nq // t))
    # shard 0 holds head 0 and the last shard holds the last head
    assert m["q_shard"][0] == 0 and m["q_shard"][nq - 1] == t - 1
    assert m["kv_shard"][0] == 0 and m["kv_shard"][nkv - 1] == t - 1
    assert m["ffn_shard"][0] == 0 and m["ffn_shard"][F - 1] == t - 1


@pytest.mark.parametrize("t", [0, 3, 5, 16, -1])
def test_plan_maps_rejects_bad_degree(t):
    assert oracle.plan_maps(oracle.Dims(256, 8, 8, 32, 64), t) is None


def test_plan_maps_rejects_indivisible():
    assert oracle.plan_maps(oracle.Dims(256, 4, 2, 64, 688), 4) is None  # 2 kv heads, t = 4
    assert oracle.plan_maps(oracle.Dims(256, 8, 8, 32, 100), 8) is None  # F = 100, t = 8


# --------------------------------------------------------------------------
# Closed forms
# --------------------------------------------------------------------------

def test_silu_known_values():
    assert oracle.silu(0.0) == 0.0
    assert oracle.silu(1.0) == pytest.approx(0.7310585786300049, abs=1e-16)
    assert oracle.silu(-1.0) == pytest.approx(-0.2689414213699951, abs=1e-16)
    assert oracle.silu(50.0) == 50.0
    assert abs(oracle.silu(-50.0)) < 1e-20


@pytest.mark.parametrize("c", [0.5, 3.0, -2.0])
def test_rmsnorm_constant_vector(c):
    n, eps = 16, 1e-5
    gamma = f32(np.linspace(0.5, 1.5, n))
    out = oracle.rmsnorm(np.full(n, c), gamma, eps)
    expect = gamma.astype(np.float64) * c / math.sqrt(c * c + eps)
    np.testing.assert_allclose(out, expect, rtol=1e-15, atol=0)


def _eye_bits(n, m=None):
    m = n if m is None else m
    e = np.zeros((n, m), np.float32)
    e[np.arange(min(n, m)), np.arange(min(n, m))] = 1
    return (e.view(np.uint32) >> 16).astype(np.uint16)


def _bits(a):
    return (f32(a).view(np.uint32) >> 16).astype(np.uint16)


def test_single_key_returns_new_value():
    """S = 0: one key, softmax weight exactly 1, so attention output = v_new."""
    r = rng(1)
    H, nq, nkv, d, F = 32, 4, 2, 8, 48
    w = small_layer(r, H, nq, nkv, d, F)
    dims = oracle.Dims(H, nq, nkv, d, F)
    x = r.standard_normal((3, H))
    kc = np.zeros((3, nkv, 4, d), np.uint16)
    y, tr = oracle.decode_layer(dims, w, x, kc, kc, 0, trace=True)
    g = nq // nkv
    for h in range(nq):
        j = h // g
        np.testing.assert_array_equal(tr["attn"][:, h * d:(h + 1) * d], tr["v_new"][:, j * d:(j + 1) * d])


def test_uniform_logits_give_mean_and_gqa_mapping():
    """Wq = 0 makes every logit 0, so each head averages its kv head's S+1
    values.  Constant, head-specific cache values pin the GQA map h -> h//g."""
    H, nq, nkv, d, F, S = 16, 8, 2, 4, 8, 5
    r = rng(2)
    w = small_layer(r, H, nq, nkv, d, F)
    w["wq"] = np.zeros_like(w["wq"])
    w["wv"] = np.zeros_like(w["wv"])           # new value = 0
    dims = oracle.Dims(H, nq, nkv, d, F, flags=0)
    B = 2
    vc = np.zeros((B, nkv, S + 3, d), np.float32)
    consts = {0: 1.5, 1: -3.0}
    for j, c in consts.items():
        vc[:, j, :S, :] = c
    kc = _bits(r.standard_normal((B, nkv, S + 3, d)))
    x = r.standard_normal((B, H))
    _, tr = oracle.decode_layer(dims, w, x, kc, _bits(vc), S, trace=True)
    g = nq // nkv
    for h in range(nq):
        np.testing.assert_allclose(tr["attn"][:, h * d:(h + 1) * d], consts[h // g] * S / (S + 1),
                                   rtol=1e-14)


def test_softmax_scale_is_inverse_sqrt_head_dim():
    """Two keys: logits (alpha*beta/sqrt(d), 0); the weight of key 0 is the
    logistic of alpha*beta/sqrt(d)."""
    d = 16
    H, nq, nkv, F = d, 1, 1, 8
    w = {"wq": _eye_bits(d), "wk": np.zeros((d, d), np.uint16), "wv": np.zeros((d, d), np.uint16),
         "wo": _eye_bits(d), "wg": np.zeros((F, H), np.uint16), "wu": np.zeros((F, H), np.uint16),
         "wd": np.zeros((H, F), np.uint16)}
    dims = oracle.Dims(H, nq, nkv, d, F, flags=0)
    alpha, beta = 2.0, 3.0
    x = np.zeros((1, H))
    x[0, 0] = beta
    kc = np.zeros((1, 1, 2, d), np.float32)
    vc = np.zeros((1, 1, 2, d), np.float32)
    kc[0, 0, 0, 0] = alpha
    vc[0, 0, 0, 1] = 1.0
    _, tr = oracle.decode_layer(dims, w, x, _bits(kc), _bits(vc), 1, trace=True)
    p0 = 1.0 / (1.0 + math.exp(-alpha * beta / math.sqrt(d)))
    assert tr["attn"][0, 1] == pytest.approx(p0, rel=1e-15)
    # Wo = I and no residual: h is the attention output itself
    np.testing.assert_array_equal(tr["h"], tr["attn"])


def test_projection_orientation_with_shift_permutations():
    """nn.Linear orientation: y = W x with W[out][in].  With cyclic-shift
    matrices a transposed product would shift the other way."""
    n = 8
    H = F = n
    d, nq, nkv = n, 1, 1
    P = np.zeros((n, n), np.float32)
    P[np.arange(n), (np.arange(n) + 1) % n] = 1      # (P x)[i] = x[i+1]
    Pb = _bits(P)
    big = _bits(np.eye(n) * 64.0)                     # gate = 64 x: silu(64 x) = 64 x for x >= 1
    w = {"wq": np.zeros((n, n), np.uint16), "wk": np.zeros((n, n), np.uint16), "wv": Pb,
         "wo": Pb, "wg": big, "wu": _eye_bits(n), "wd": Pb}
    dims = oracle.Dims(H, nq, nkv, d, F, flags=oracle.RESIDUAL)
    x = np.arange(1, n + 1, dtype=np.float64)[None] * 1.0
    y, tr = oracle.decode_layer(dims, w, x, np.zeros((1, 1, 1, d), np.uint16),
                                np.zeros((1, 1, 1, d), np.uint16), 0, trace=True)
    sh = lambda v, k: np.roll(v, -k, axis=-1)
    np.testing.assert_array_equal(tr["v_new"], sh(x, 1))          # Wv x
    np.testing.assert_array_equal(tr["attn"], sh(x, 1))           # single key
    np.testing.assert_array_equal(tr["h"], x + sh(x, 2))          # x + Wo attn
    m = tr["h"]
    act = (64.0 * m) * m                                           # silu(64 m) * m
    np.testing.assert_allclose(y, m + sh(act, 1), rtol=1e-15)


def test_swiglu_identity_weights():
    """Wg = Wu = Wd = I, Wo = 0, no norm: h = x and y = x + silu(x) * x."""
    n = 16
    w = {"wq": np.zeros((n, n), np.uint16), "wk": np.zeros((n, n), np.uint16),
         "wv": np.zeros((n, n), np.uint16), "wo": np.zeros((n, n), np.uint16),
         "wg": _eye_bits(n), "wu": _eye_bits(n), "wd": _eye_bits(n)}
    dims = oracle.Dims(n, 1, 1, n, n, flags=oracle.RESIDUAL)
    x = np.linspace(-4, 4, n)[None]
    y, tr = oracle.decode_layer(dims, w, x, np.zeros((1, 1, 1, n), np.uint16),
                                np.zeros((1, 1, 1, n), np.uint16), 0, trace=True)
    np.testing.assert_array_equal(tr["h"], x)
    np.testing.assert_allclose(tr["act"][0], x[0] * x[0] / (1 + np.exp(-x[0])), rtol=1e-15)
    np.testing.assert_allclose(y[0], x[0] + x[0] * x[0] / (1 + np.exp(-x[0])), rtol=1e-15)


def test_residuals_with_zero_branches():
    r = rng(3)
    H, nq, nkv, d, F = 16, 2, 1, 8, 24
    w = small_layer(r, H, nq, nkv, d, F)
    w["wo"] = np.zeros_like(w["wo"])
    w["wg"] = np.zeros_like(w["wg"])
    x = r.standard_normal((2, H))
    dims = oracle.Dims(H, nq, nkv, d, F)
    kc = rand_bf16_bits(r, (2, nkv, 5, d), 1.0)
    y, tr = oracle.decode_layer(dims, w, x, kc, kc, 3, trace=True)
    np.testing.assert_array_equal(tr["h"], x)
    np.testing.assert_array_equal(y, x)


# --------------------------------------------------------------------------
# Exact row-split / column-split identities (integer data, every sum exact)
# --------------------------------------------------------------------------

@pytest.mark.parametrize("t", [1, 2, 4, 8])
def test_mlp_row_split_identity_exact(t):
    """Sum of the t row-split partials equals the unsharded MLP bit for bit.
    Gate inputs are >= 40 so silu(g) == g exactly in float64 and every value
    is an integer."""
    r = rng(10 + t)
    H, F, B = 8, 16, 3
    x = r.integers(5, 9, (B, H)).astype(np.float64)
    wg = f32(r.integers(1, 9, (F, H)))
    wu = f32(r.integers(-8, 9, (F, H)))
    wd = f32(r.integers(-8, 9, (H, F)))
    z = np.zeros((4, H), np.float32)
    w = {"wq": z, "wk": z, "wv": z, "wo": f32(np.zeros((H, 4))), "wg": wg, "wu": wu, "wd": wd}
    dims = oracle.Dims(H, 1, 1, 4, F, flags=oracle.RESIDUAL)
    kc = np.zeros((B, 1, 1, 4), np.uint16)
    # wo = 0 makes h = x, so the layer is x + MLP(x); every value is an integer
    y_full = oracle.decode_layer(dims, w, x, kc, kc, 0) - x
    y_sh, parts = oracle.mlp_sharded(dims, w, t, x, partials=True)
    np.testing.assert_array_equal(y_sh, y_full)
    np.testing.assert_array_equal(parts.sum(axis=0), y_full)
    # and against exact integer arithmetic
    g = x @ wg.T.astype(np.float64)
    assert np.all(g >= 40)
    exact = (g * (x @ wu.T.astype(np.float64))) @ wd.T.astype(np.float64)
    np.testing.assert_array_equal(y_full, exact)


@pytest.mark.parametrize("t", [1, 2, 4, 8])
def test_attention_head_split_identity_exact(t):
    """S = 0 and integer data: attention output = v exactly; the head-wise
    column split plus row-split O projection sums to the unsharded h."""
    r = rng(20 + t)
    H, nq, nkv, d, B = 16, 8, 8, 4, 2
    w = {"wq": f32(r.integers(-8, 9, (nq * d, H))), "wk": f32(r.integers(-8, 9, (nkv * d, H))),
         "wv": f32(r.integers(-8, 9, (nkv * d, H))), "wo": f32(r.integers(-8, 9, (H, nq * d))),
         "wg": f32(np.zeros((4, H))), "wu": f32(np.zeros((4, H))), "wd": f32(np.zeros((H, 4)))}
    dims = oracle.Dims(H, nq, nkv, d, 4, flags=oracle.RESIDUAL)
    x = r.integers(-8, 9, (B, H)).astype(np.float64)
    kc = np.zeros((B, nkv, 2, d), np.uint16)
    _, tr = oracle.decode_layer(dims, w, x, kc, kc, 0, trace=True)
    h_sh, parts = oracle.attn_sharded(dims, w, t, x, x, kc, kc, 0, partials=True)
    np.testing.assert_array_equal(h_sh, tr["h"])
    exact = x + (x @ w["wv"].T.astype(np.float64)) @ w["wo"].T.astype(np.float64)
    np.testing.assert_array_equal(tr["h"], exact)


@pytest.mark.parametrize("t", [1, 2, 4])
def test_attention_head_split_identity_gqa(t):
    """GQA with a real cache: sharded and unsharded agree to rounding."""
    r = rng(30 + t)
    H, nq, nkv, d, F, B, S = 32, 8, 4, 8, 16, 2, 7
    w = small_layer(r, H, nq, nkv, d, F)
    dims = oracle.Dims(H, nq, nkv, d, F, flags=oracle.NORM | oracle.RESIDUAL)
    x = r.standard_normal((B, H))
    kc = rand_bf16_bits(r, (B, nkv, S + 2, d), 1.0)
    vc = rand_bf16_bits(r, (B, nkv, S + 2, d), 1.0)
    _, tr = oracle.decode_layer(dims, w, x, kc, vc, S, trace=True)
    a = np.stack([oracle.rmsnorm(x[b], w["gamma_attn"], dims.eps) for b in range(B)])
    h_sh = oracle.attn_sharded(dims, w, t, x, a, kc, vc, S)
    np.testing.assert_allclose(h_sh, tr["h"], rtol=1e-12, atol=1e-12)


# --------------------------------------------------------------------------
# Independent evaluation with numpy's library routines
# --------------------------------------------------------------------------

@pytest.mark.parametrize("case", [
    dict(H=256, nq=4, nkv=2, d=64, F=688, B=1, S=0, flags=0),          # MLP-shaped tiny case
    dict(H=64, nq=4, nkv=4, d=16, F=96, B=3, S=9, flags=3),             # MHA, g = 1
    dict(H=64, nq=8, nkv=2, d=16, F=80, B=2, S=33, flags=3),            # GQA, g = 4
    dict(H=32, nq=4, nkv=1, d=8, F=40, B=2, S=5, flags=1),              # norm only
])
def test_decode_matches_numpy(case):
    r = rng(40)
    H, nq, nkv, d, F, B, S = (case[k] for k in ("H", "nq", "nkv", "d", "F", "B", "S"))
    w = small_layer(r, H, nq, nkv, d, F, std=0.1)
    dims = oracle.Dims(H, nq, nkv, d, F, flags=case["flags"])
    x = r.standard_normal((B, H))
    kc = rand_bf16_bits(r, (B, nkv, S + 4, d), 1.0)
    vc = rand_bf16_bits(r, (B, nkv, S + 4, d), 1.0)
    y, tr = oracle.decode_layer(dims, w, x, kc, vc, S, trace=True)
    y_np, tr_np = np_reference.decode_layer(H, nq, nkv, d, F, dims.eps, bool(dims.flags & 1),
                                            bool(dims.flags & 2), w, x, kc, vc, S)
    scale = np.abs(y_np).max()
    np.testing.assert_allclose(y, y_np, rtol=1e-12, atol=1e-12 * scale)
    for k in tr:
        s = max(np.abs(tr_np[k]).max(), 1e-300)
        np.testing.assert_allclose(tr[k], tr_np[k], rtol=1e-12, atol=1e-12 * s)


def test_decode_fp32_weights_match_numpy():
    r = rng(41)
    H, nq, nkv, d, F, B, S = 64, 8, 2, 16, 80, 2, 12
    w = small_layer(r, H, nq, nkv, d, F, std=0.1, bf16=False)
    dims = oracle.Dims(H, nq, nkv, d, F)
    x = r.standard_normal((B, H))
    kc = rand_bf16_bits(r, (B, nkv, S + 1, d), 1.0)
    vc = rand_bf16_bits(r, (B, nkv, S + 1, d), 1.0)
    y = oracle.decode_layer(dims, w, x, kc, vc, S)
    y_np, _ = np_reference.decode_layer(H, nq, nkv, d, F, dims.eps, True, True, w, x, kc, vc, S)
    np.testing.assert_allclose(y, y_np, rtol=1e-12, atol=1e-12 * np.abs(y_np).max())


def test_prefill_matches_numpy():
    r = rng(42)
    H, nq, nkv, d, F, T = 64, 8, 2, 16, 80, 13
    w = small_layer(r, H, nq, nkv, d, F, std=0.1)
    dims = oracle.Dims(H, nq, nkv, d, F)
    x = r.standard_normal((T, H))
    y, k, v = oracle.prefill_layer(dims, w, x)
    y_np, k_np, v_np = np_reference.prefill_layer(H, nq, nkv, d, F, dims.eps, True, True, w, x)
    np.testing.assert_allclose(y, y_np, rtol=1e-12, atol=1e-12 * np.abs(y_np).max())
    np.testing.assert_allclose(k, k_np, rtol=1e-12, atol=1e-12 * np.abs(k_np).max())


def test_prefill_is_causal_and_agrees_with_decode():
    """Token i of a prefill chunk sees only tokens 0..i: changing later tokens
    leaves earlier outputs unchanged, and with bf16-exact keys/values the last
    token equals one decode step over a cache holding the earlier tokens."""
    r = rng(43)
    H, nq, nkv, d, F, T = 16, 4, 2, 8, 12, 6
    w = {k: f32(r.integers(-2, 3, s)) for k, s in
         {"wq": (nq * d, H), "wk": (nkv * d, H), "wv": (nkv * d, H), "wo": (H, nq * d),
          "wg": (F, H), "wu": (F, H), "wd": (H, F)}.items()}
    w["wq"] = f32(w["wq"] * 0.125)
    dims = oracle.Dims(H, nq, nkv, d, F, flags=oracle.RESIDUAL)
    x = r.integers(-2, 3, (T, H)).astype(np.float64)
    y, k, v = oracle.prefill_layer(dims, w, x)
    x2 = x.copy()
    x2[-1] += 1.0
    y2, _, _ = oracle.prefill_layer(dims, w, x2)
    np.testing.assert_array_equal(y[:-1], y2[:-1])
    assert not np.array_equal(y[-1], y2[-1])
    # keys and values are small integers: exact in bf16
    S = T - 1
    kc = np.zeros((1, nkv, T, d), np.float32)
    vc = np.zeros((1, nkv, T, d), np.float32)
    for j in range(nkv):
        kc[0, j, :S] = k[:S, j * d:(j + 1) * d]
        vc[0, j, :S] = v[:S, j * d:(j + 1) * d]
    assert np.array_equal(_bits(kc).astype(np.uint32) << 16, kc.view(np.uint32))
    yd = oracle.decode_layer(dims, w, x[-1:], _bits(kc), _bits(vc), S)
    np.testing.assert_allclose(yd[0], y[-1], rtol=1e-13, atol=1e-13)
    # token 0 of the chunk is a decode step over an empty cache
    y0 = oracle.decode_layer(dims, w, x[:1], np.zeros((1, nkv, 1, d), np.uint16),
                             np.zeros((1, nkv, 1, d), np.uint16), 0)
    np.testing.assert_allclose(y0[0], y[0], rtol=1e-14, atol=1e-14)


# --------------------------------------------------------------------------
# Planted mistakes must be caught (a check of the checks, done on the CPU)
# --------------------------------------------------------------------------

def test_planted_transposed_wo_is_caught():
    """A transposed O projection in a reference would fail the orientation
    pin: emulate it with numpy and confirm the pinned values differ."""
    n = 8
    P = np.zeros((n, n))
    P[np.arange(n), (np.arange(n) + 1) % n] = 1
    o = np.arange(1, n + 1, dtype=np.float64)
    assert not np.array_equal(P @ o, P.T @ o)


def test_prefill_rows_match_the_whole_chunk():
    """The sampled-row form gives, at each listed row (any order, repeats
    allowed), the whole chunk's row; keys/values up to the last listed row."""
    r = rng(47)
    H, nq, nkv, d, F, T = 32, 4, 2, 8, 24, 9
    w = small_layer(r, H, nq, nkv, d, F)
    dims = oracle.Dims(H, nq, nkv, d, F)
    x = r.normal(0, 1, (T, H))
    y, k, v, tr = oracle.prefill_layer(dims, w, x, trace=True)
    rows = [6, 0, 3, 6]
    ys, ks, vs, trs = oracle.prefill_rows(dims, w, x, rows, trace=True)
    np.testing.assert_array_equal(ys, y[rows])
    np.testing.assert_array_equal(ks, k[:7])
    np.testing.assert_array_equal(vs, v[:7])
    for name in ("q", "attn", "h", "act"):
        np.testing.assert_array_equal(trs[name], tr[name][rows])
    with pytest.raises(ValueError):
        oracle.prefill_rows(dims, w, x, [T])


# --------------------------------------------------------------------------
# Rotary position embedding and chunked prefill into an existing cache
# --------------------------------------------------------------------------

@pytest.mark.parametrize("d,base", [(8, 10000.0), (128, 500000.0), (128, 10000.0)])
def test_rope_matches_complex_rotation(d, base):
    r = rng(60)
    v = r.standard_normal((5, d))
    for pos in (0, 1, 7, 4096, 8191, 131071):
        got = oracle.rope(v, pos, base)
        want = np_reference.rope(v, pos, base)
        # the angle pos * theta carries a rounding of about pos * 1e-16 rad
        np.testing.assert_allclose(got, want, rtol=0, atol=(1e-14 + 1e-15 * pos) * np.abs(v).max())


def test_rope_invariants():
    r = rng(61)
    d, base = 128, 500000.0
    q, k = r.standard_normal(d), r.standard_normal(d)
    # position 0 is the identity, exactly
    np.testing.assert_array_equal(oracle.rope(q, 0, base), q)
    # each pair (e, e + d/2) keeps its length
    for pos in (1, 33, 8000):
        rq = oracle.rope(q, pos, base)
        np.testing.assert_allclose(rq[:64] ** 2 + rq[64:] ** 2, q[:64] ** 2 + q[64:] ** 2, rtol=1e-12)
    # the logit depends on the distance only: <R(m) q, R(n) k> = <R(m+c) q, R(n+c) k>
    for m, n, c in ((5, 2, 100), (0, 9, 4000), (8191, 0, 7)):
        a = oracle.rope(q, m, base) @ oracle.rope(k, n, base)
        b = oracle.rope(q, m + c, base) @ oracle.rope(k, n + c, base)
        assert abs(a - b) <= 1e-10 * np.abs(q).sum() * np.abs(k).max()
    # pair 0 turns by exactly pos radians (theta_0 = 1); the last pair slowest
    e0 = np.zeros(d)
    e0[0] = 1.0
    rq = oracle.rope(e0, 3, base)
    assert rq[0] == pytest.approx(np.cos(3.0), abs=1e-15) and rq[64] == pytest.approx(np.sin(3.0), abs=1e-15)
    e1 = np.zeros(d)
    e1[63] = 1.0
    rq = oracle.rope(e1, 3, base)
    ang = 3.0 * base ** (-126.0 / 128.0)
    assert rq[63] == pytest.approx(np.cos(ang), abs=1e-15) and rq[127] == pytest.approx(np.sin(ang), abs=1e-15)


@pytest.mark.parametrize("rope", [False, True])
def test_decode_with_rope_matches_numpy(rope):
    r = rng(62)
    H, nq, nkv, d, F, B, S = 64, 8, 2, 16, 80, 2, 11
    w = small_layer(r, H, nq, nkv, d, F, std=0.1)
    flags = oracle.NORM | oracle.RESIDUAL | (oracle.ROPE if rope else 0)
    dims = oracle.Dims(H, nq, nkv, d, F, flags=flags, rope_base=10000.0)
    x = r.standard_normal((B, H))
    kc = rand_bf16_bits(r, (B, nkv, S + 2, d), 1.0)
    vc = rand_bf16_bits(r, (B, nkv, S + 2, d), 1.0)
    y, tr = oracle.decode_layer(dims, w, x, kc, vc, S, trace=True)
    y_np, tr_np = np_reference.decode_layer(H, nq, nkv, d, F, dims.eps, True, True, w, x, kc, vc, S,
                                            rope_base=10000.0 if rope else None)
    np.testing.assert_allclose(y, y_np, rtol=1e-11, atol=1e-11 * np.abs(y_np).max())
    np.testing.assert_allclose(tr["q"], tr_np["q"], rtol=1e-11, atol=1e-11 * np.abs(tr_np["q"]).max())
    np.testing.assert_allclose(tr["k_new"], tr_np["k_new"], rtol=1e-11,
                               atol=1e-11 * np.abs(tr_np["k_new"]).max())


@pytest.mark.parametrize("rope,P0", [(False, 0), (False, 9), (True, 0), (True, 9), (True, 300)])
def test_prefill_chunk_matches_numpy(rope, P0):
    r = rng(63)
    H, nq, nkv, d, F, T = 64, 8, 2, 16, 80, 7
    w = small_layer(r, H, nq, nkv, d, F, std=0.1)
    flags = oracle.NORM | oracle.RESIDUAL | (oracle.ROPE if rope else 0)
    dims = oracle.Dims(H, nq, nkv, d, F, flags=flags, rope_base=500000.0)
    x = r.standard_normal((T, H))
    kc = rand_bf16_bits(r, (nkv, P0 + T + 3, d), 1.0)
    vc = rand_bf16_bits(r, (nkv, P0 + T + 3, d), 1.0)
    y, k, v = oracle.prefill_chunk(dims, w, x, P0, kc, vc)
    y_np, k_np, v_np = np_reference.prefill_layer(H, nq, nkv, d, F, dims.eps, True, True, w, x, P0, kc, vc,
                                                  rope_base=500000.0 if rope else None)
    np.testing.assert_allclose(y, y_np, rtol=1e-11, atol=1e-11 * np.abs(y_np).max())
    np.testing.assert_allclose(k, k_np, rtol=1e-11, atol=1e-11 * np.abs(k_np).max())
    np.testing.assert_allclose(v, v_np, rtol=1e-11, atol=1e-11 * np.abs(v_np).max())


@pytest.mark.parametrize("rope", [False, True])
def test_one_token_chunk_is_a_decode_step(rope):
    """A chunk of one token at position S over a cache of S tokens is the
    decode step at S (the same definition reached by two routes)."""
    r = rng(64)
    H, nq, nkv, d, F, S = 32, 4, 2, 8, 24, 13
    w = small_layer(r, H, nq, nkv, d, F)
    flags = oracle.NORM | oracle.RESIDUAL | (oracle.ROPE if rope else 0)
    dims = oracle.Dims(H, nq, nkv, d, F, flags=flags, rope_base=10000.0)
    x = r.standard_normal((1, H))
    kc = rand_bf16_bits(r, (1, nkv, S + 1, d), 1.0)
    vc = rand_bf16_bits(r, (1, nkv, S + 1, d), 1.0)
    yd, trd = oracle.decode_layer(dims, w, x, kc, vc, S, trace=True)
    yc, kk, vv, trc = oracle.prefill_chunk(dims, w, x, S, kc, vc, trace=True)
    np.testing.assert_allclose(yc, yd, rtol=1e-13, atol=1e-13 * np.abs(yd).max())
    np.testing.assert_allclose(kk, trd["k_new"], rtol=1e-14, atol=0)
    np.testing.assert_allclose(trc["attn"], trd["attn"], rtol=1e-13, atol=1e-13 * np.abs(trd["attn"]).max())


def test_chunks_compose_to_the_whole_sequence():
    """With keys and values exact in bf16 (small integers), prefilling a
    sequence in two chunks (the second attending to the first's cached keys)
    gives the single chunk's outputs."""
    r = rng(65)
    H, nq, nkv, d, F, T1, T2 = 16, 4, 2, 8, 12, 5, 4
    w = {k: f32(r.integers(-2, 3, s)) for k, s in
         {"wq": (nq * d, H), "wk": (nkv * d, H), "wv": (nkv * d, H), "wo": (H, nq * d),
          "wg": (F, H), "wu": (F, H), "wd": (H, F)}.items()}
    w["wq"] = f32(w["wq"] * 0.125)
    dims = oracle.Dims(H, nq, nkv, d, F, flags=oracle.RESIDUAL)
    x = r.integers(-2, 3, (T1 + T2, H)).astype(np.float64)
    y, k, v = oracle.prefill_layer(dims, w, x)
    y1, k1, v1 = oracle.prefill_chunk(dims, w, x[:T1], 0)
    kc = np.zeros((nkv, T1 + T2, d), np.float32)
    vc = np.zeros((nkv, T1 + T2, d), np.float32)
    for j in range(nkv):
        kc[j, :T1] = k1[:, j * d:(j + 1) * d]
        vc[j, :T1] = v1[:, j * d:(j + 1) * d]
    assert np.array_equal(_bits(kc).astype(np.uint32) << 16, kc.view(np.uint32))  # exact in bf16
    y2, k2, v2 = oracle.prefill_chunk(dims, w, x[T1:], T1, _bits(kc), _bits(vc))
    np.testing.assert_allclose(np.concatenate([y1, y2]), y, rtol=1e-13, atol=1e-13 * np.abs(y).max())
    np.testing.assert_array_equal(np.concatenate([k1, k2]), k)
    # a changed prefix changes the second chunk (it is read), a changed later
    # token does not change the first
    kc2 = kc.copy()
    kc2[0, 0, 0] += 1.0
    y2b, _, _ = oracle.prefill_chunk(dims, w, x[T1:], T1, _bits(kc2), _bits(vc))
    assert not np.array_equal(y2b, y2)
    with pytest.raises(ValueError):
        oracle.prefill_chunk(dims, w, x[T1:], T1)  # a prefix needs a cache


# --------------------------------------------------------------------------
# Planner extras: Auto shard degree and the TP cost model
# --------------------------------------------------------------------------

D70 = (8192, 64, 8, 128, 28672)


def test_scaling_math_worked_example():
    """The pages' TP=2 example: 160 calls at 8 us, 30 ms -> 16.3 ms, 1.84x."""
    g = golden("scaling_math.json")
    comm = oracle.tp_time(0.0, g["n"], g["layers"], g["t_allreduce_s"])
    assert comm == pytest.approx(2 * g["layers"] * g["t_allreduce_s"], rel=1e-15)
    assert abs(comm - g["comm_s_approx"]) <= 0.05e-3  # 1.28 ms, printed as about 1.3
    tn = oracle.tp_time(g["t_single_s"], g["n"], g["layers"], g["t_allreduce_s"])
    assert abs(tn - g["t_n_s_approx"]) <= 0.05e-3
    assert abs(g["t_single_s"] / tn - g["speedup_approx"]) <= 0.005
    # no exchange at N = 1: T(1) is the single-GPU time
    assert oracle.tp_time(g["t_single_s"], 1, g["layers"], 0.0) == g["t_single_s"]


def test_allreduce_time_closed_forms():
    g = golden("scaling_math.json")
    m, lat, bw = g["message_bytes"], 7e-6, 770e9
    assert oracle.allreduce_time(1, m, lat, bw) == 0.0
    # ring: 2 (N-1)/N of the message crosses each link
    for n in (2, 4, 8):
        assert oracle.allreduce_time(n, m, lat, bw) == pytest.approx(lat + 2 * (n - 1) / n * m / bw, rel=1e-15)
    assert oracle.allreduce_time(2, m, lat, bw) == pytest.approx(lat + m / bw, rel=1e-15)
    # a 16 KB message: the latency dominates (the bandwidth part is a few ns)
    for n in (2, 4, 8):
        t = oracle.allreduce_time(n, m, lat, bw)
        assert g["latency_range_s"][0] <= t <= g["latency_range_s"][1]
        assert (t - lat) < 0.01 * lat
    # bandwidth-bound limit: latency 0, huge message -> 2 (N-1)/N * M / bw
    assert oracle.allreduce_time(8, 1 << 30, 0.0, bw) == pytest.approx(1.75 * (1 << 30) / bw, rel=1e-15)


def test_footprint_per_gpu_is_weights_plus_kv():
    d = oracle.Dims(*D70)
    for t in (1, 2, 4, 8):
        w = 80 * oracle.layer_params_per_shard(d, t) * 2
        kv = oracle.kv_bytes_per_shard(80, 8, 128, 8192, 2, 16, t)
        assert oracle.footprint_per_gpu(d, 80, t, 16, 8192) == w + kv
    assert oracle.footprint_per_gpu(d, 80, 3, 16, 8192) == -1  # 3 divides no head count
    assert oracle.footprint_per_gpu(d, 80, 16, 16, 8192) == -1  # more shards than kv heads


def test_auto_t_70b_on_80gb_cards():
    """Auto on the pages' 70B example: t = 4 is the smallest that fits."""
    g = golden("auto_t.json")
    d = oracle.Dims(*D70)
    t = oracle.auto_t(d, 80, g["gpu_bytes"], g["headroom"], g["batch"], g["seq"])
    assert t == g["expected_t"]
    # t = 2 misses (about 90 GB per GPU), t = 4 fits (about 45 GB)
    assert oracle.footprint_per_gpu(d, 80, 2, 16, 8192) > g["gpu_bytes"]
    assert oracle.footprint_per_gpu(d, 80, 4, 16, 8192) < g["gpu_bytes"] * (1 - g["headroom"])


def test_auto_t_prefers_one_and_powers_of_two():
    d7 = oracle.Dims(4096, 32, 32, 128, 11008)
    # a 7B layer stack fits a 180 GB card alone
    assert oracle.auto_t(d7, 32, 180 * 10**9, 0.1, 1, 2048) == 1
    # a budget between two footprints picks the first power of two above it
    f = {t: oracle.footprint_per_gpu(d7, 32, t, 64, 4096) for t in (1, 2, 4, 8)}
    assert f[1] > f[2] > f[4] > f[8]
    for t in (1, 2, 4, 8):
        assert oracle.auto_t(d7, 32, f[t], 0.0, 64, 4096) == t
        assert oracle.auto_t(d7, 32, f[t] - 1, 0.0, 64, 4096) == (2 * t if t < 8 else 0)
    # headroom: exactly at budget * (1 - h) still fits, one byte more does not
    h = 0.25
    b = int(f[2] / (1 - h))
    while b * (1 - h) < f[2]:
        b += 1
    assert oracle.auto_t(d7, 32, b, h, 64, 4096) == 2
    # nothing fits: 0
    assert oracle.auto_t(d7, 32, 1000, 0.0, 64, 4096) == 0
    # max_t caps the search
    assert oracle.auto_t(d7, 32, f[8], 0.0, 64, 4096, max_t=4) == 0


def test_auto_t_blind_fallback_and_divisibility():
    d70 = oracle.Dims(*D70)
    # memory unknown: the largest power of two the GPU count allows
    for gpus, want in ((1, 1), (2, 2), (3, 2), (4, 4), (7, 4), (8, 8), (16, 8)):
        assert oracle.auto_t(d70, 80, 0, 0.1, 16, 8192, max_t=gpus) == want
    # 2 kv heads: t = 4 and 8 do not divide, so the blind answer stops at 2
    d = oracle.Dims(1024, 16, 2, 64, 2816)
    assert oracle.auto_t(d, 4, 0, 0.0, 1, 16, max_t=8) == 2
    # a budget only t = 4 would meet is not met by any admissible t
    f4 = oracle.footprint_per_gpu(oracle.Dims(1024, 16, 4, 64, 2816), 4, 4, 1, 16)
    assert oracle.auto_t(d, 4, f4, 0.0, 1, 16) == 0
