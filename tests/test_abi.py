"""Host-side checks of the C-ABI library: it loads, exports every symbol the
header declares, and its planner agrees bit-exactly with the oracle's own
derivation of the shard maps and footprints.  No GPU needed: nothing here
launches a kernel."""
import ctypes
import json
import os
import re

import numpy as np
import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def tpl():
    from megatron_tensor_transformer_plan_b200 import build
    build.build()
    from megatron_tensor_transformer_plan_b200 import tpl as m
    return m


def header_functions():
    text = open(os.path.join(ROOT, "include", "tpl.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(tpl_[a-z_0-9]+)\s*\(", text)))


def test_exports_every_declared_function(tpl):
    names = header_functions()
    assert len(names) >= 20
    lib = ctypes.CDLL(tpl.LIB_PATH)
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing


CONFIGS = [
    # (H, nq, nkv, d, F, L)
    (256, 2, 2, 128, 688, 1),          # tiny MLP block
    (4096, 32, 32, 128, 11008, 32),    # 7B-shaped
    (8192, 64, 8, 128, 28672, 80),     # 70B-shaped
]


@pytest.mark.parametrize("cfg", CONFIGS)
@pytest.mark.parametrize("t", [1, 2, 4, 8])
def test_maps_match_oracle(tpl, cfg, t):
    H, nq, nkv, d, F, L = cfg
    dims = tpl.make_dims(H, nq, nkv, d, F, L)
    od = oracle.Dims(H, nq, nkv, d, F)
    ref = oracle.plan_maps(od, t)
    h = ctypes.c_void_p()
    rc = tpl.tpl_plan_create(ctypes.byref(dims), t, ctypes.byref(h))
    if ref is None:
        assert rc == tpl.TPL_EINDIVISIBLE
        return
    assert rc == tpl.TPL_OK
    tpl.tpl_plan_destroy(h)
    plan = tpl.Plan(dims, t)
    m = plan.maps()
    for k in ("q_shard", "q_local", "kv_shard", "ffn_shard"):
        np.testing.assert_array_equal(m[k], ref[k], err_msg=k)
    info = plan.info()
    assert info.layer_params_per_shard == oracle.layer_params_per_shard(od, t)
    assert info.layer_weight_bytes_per_shard == 2 * info.layer_params_per_shard
    assert info.reductions_per_step == oracle.reductions_per_pass(L)
    assert info.q_heads_per_shard == nq // t and info.kv_heads_per_shard == nkv // t
    assert info.ffn_per_shard == F // t
    # the packed blocks tile the packed layer without overlap
    offs = m["packed_offsets"]
    assert np.all(np.diff(offs) > 0) and offs[-1] < info.packed_layer_bytes
    assert np.all(offs % 256 == 0)


def test_70b_numbers(tpl):
    plan = tpl.Plan(tpl.make_dims(8192, 64, 8, 128, 28672, 80), 4)
    info = plan.info()
    assert info.layer_params_per_shard == 213_909_504
    assert info.qkv_rows_per_shard == (16 + 2 * 2) * 128
    plan8 = tpl.Plan(tpl.make_dims(8192, 64, 8, 128, 28672, 80), 8)
    assert plan8.info().layer_params_per_shard == 106_954_752
    assert plan8.info().reductions_per_step == 160


def test_kv_bytes_worked_example(tpl):
    g = json.load(open(os.path.join(ROOT, "tests", "golden", "kv_footprint.json")))
    dims = tpl.make_dims(8192, 64, g["kv_heads"], g["head_dim"], 28672, g["layers"])
    assert tpl.tpl_kv_bytes(ctypes.byref(dims), 1, 1, g["seq"], g["bytes_per_elem"]) == g["bytes_per_sequence"]
    assert tpl.tpl_kv_bytes(ctypes.byref(dims), 1, g["batch"], g["seq"], g["bytes_per_elem"]) == g["bytes_batch"]
    assert tpl.tpl_kv_bytes(ctypes.byref(dims), g["t"], g["batch"], g["seq"], g["bytes_per_elem"]) == g["bytes_per_gpu"]
    for t in (1, 2, 4, 8):
        for B, S in ((1, 1), (4, 4096), (16, 8192), (3, 777)):
            assert tpl.tpl_kv_bytes(ctypes.byref(dims), t, B, S, 2) == \
                oracle.kv_bytes_per_shard(80, 8, 128, S, 2, B, t)
    assert tpl.tpl_kv_bytes(ctypes.byref(dims), 0, 1, 1, 2) == -1


def test_kv_layer_bytes_matches_per_gpu_formula(tpl):
    plan = tpl.Plan(tpl.make_dims(8192, 64, 8, 128, 28672, 80), 4)
    # all shards of one layer = t * (per-GPU bytes of one layer)
    per_gpu_one_layer = oracle.kv_bytes_per_shard(1, 8, 128, 8192, 2, 16, 4)
    assert 2 * plan.kv_layer_bytes(16, 8192) == 4 * per_gpu_one_layer


@pytest.mark.parametrize("t,code", [(3, 2), (0, 2), (16, 2), (-1, 2)])
def test_plan_rejects_bad_degree(tpl, t, code):
    dims = tpl.make_dims(256, 8, 8, 128, 64)
    h = ctypes.c_void_p()
    assert tpl.tpl_plan_create(ctypes.byref(dims), t, ctypes.byref(h)) == code
    assert not h.value


def test_plan_rejects_bad_dims(tpl):
    h = ctypes.c_void_p()
    cases = [
        (tpl.make_dims(256, 4, 2, 128, 688), 4, tpl.TPL_EINDIVISIBLE),   # t does not divide n_kv
        (tpl.make_dims(256, 6, 4, 128, 688), 1, tpl.TPL_EINDIVISIBLE),   # n_kv does not divide n_q
        (tpl.make_dims(256, 4, 4, 64, 688), 1, tpl.TPL_EUNSUPPORTED),    # head_dim 64
        (tpl.make_dims(256, 64, 2, 128, 688), 1, tpl.TPL_EUNSUPPORTED),  # group of 32
        (tpl.make_dims(250, 4, 4, 128, 688), 1, tpl.TPL_EUNSUPPORTED),   # hidden % 8
        (tpl.make_dims(0, 4, 4, 128, 688), 1, tpl.TPL_EINVAL),
        (tpl.make_dims(256, 4, 4, 128, 688, flags=64), 1, tpl.TPL_EINVAL),
    ]
    for dims, t, code in cases:
        assert tpl.tpl_plan_create(ctypes.byref(dims), t, ctypes.byref(h)) == code, (dims.hidden, t)
    assert tpl.tpl_plan_create(None, 1, ctypes.byref(h)) == tpl.TPL_EINVAL
    dims = tpl.make_dims(256, 4, 4, 128, 688)
    assert tpl.tpl_plan_create(ctypes.byref(dims), 1, None) == tpl.TPL_EINVAL


def test_device_calls_validate_before_launch(tpl):
    """Host validation returns a status without touching the GPU (this box has
    none, so any launch attempt would report TPL_ECUDA instead)."""
    plan = tpl.Plan(tpl.make_dims(256, 2, 2, 128, 688), 2)
    need = plan.workspace_size(1, 0)
    fake = 1 << 20  # an aligned, never dereferenced address
    kv = tpl.tpl_kv(fake, fake, 1, 16)
    H = plan.handle
    st = None
    # null workspace
    assert tpl.tpl_decode_layer(H, fake, ctypes.byref(kv), fake, 1, 0, fake, None, None, need, 0, st) == tpl.TPL_EINVAL
    # workspace too small
    assert tpl.tpl_decode_layer(H, fake, ctypes.byref(kv), fake, 1, 0, fake, None, fake, need - 1, 0, st) == \
        tpl.TPL_EWORKSPACE
    # batch beyond what the decode kernels take: 64 tokens (16 with fp32 weights)
    assert tpl.tpl_decode_layer(H, fake, ctypes.byref(kv), fake, 65, 0, fake, None, fake, 1 << 40, 0, st) == \
        tpl.TPL_EUNSUPPORTED
    assert tpl.tpl_decode_layer(H, fake, ctypes.byref(kv), fake, 17, 0, fake, None, fake, 1 << 40, 0, st) == \
        tpl.TPL_ENOMEM  # supported; the cache holds one sequence
    p32 = tpl.Plan(tpl.make_dims(256, 2, 2, 128, 688, 1, 1e-5, tpl.TPL_FP32_WEIGHTS), 2)
    assert tpl.tpl_decode_layer(p32.handle, fake, ctypes.byref(kv), fake, 17, 0, fake, None, fake, 1 << 40, 0,
                                st) == tpl.TPL_EUNSUPPORTED
    # KV capacity: S must be < seq_cap, B <= batch_cap
    assert tpl.tpl_decode_layer(H, fake, ctypes.byref(kv), fake, 1, 16, fake, None, fake, 1 << 40, 0, st) == \
        tpl.TPL_ENOMEM
    assert tpl.tpl_decode_layer(H, fake, ctypes.byref(kv), fake, 2, 0, fake, None, fake, 1 << 40, 0, st) == \
        tpl.TPL_ENOMEM
    # misaligned activation pointer
    assert tpl.tpl_decode_layer(H, fake, ctypes.byref(kv), fake + 2, 1, 0, fake, None, fake, 1 << 40, 0, st) == \
        tpl.TPL_EINVAL
    # bad reduce mode
    assert tpl.tpl_decode_layer(H, fake, ctypes.byref(kv), fake, 1, 0, fake, None, fake, 1 << 40, 7, st) == \
        tpl.TPL_EINVAL
    # packing into a buffer that is too small
    w = tpl.tpl_layer_weights(fake, fake, fake, fake, fake, fake, fake, None, None)
    assert tpl.tpl_pack_layer(H, ctypes.byref(w), fake, 10, st) == tpl.TPL_ENOMEM
    # B == 0 is a no-op
    assert tpl.tpl_decode_layer(H, fake, ctypes.byref(kv), fake, 0, 0, fake, None, None, 0, 0, st) == tpl.TPL_OK
    assert tpl.tpl_status_string(tpl.TPL_EWORKSPACE) == b"workspace too small"


def test_workspace_grows_with_batch_and_length(tpl):
    plan = tpl.Plan(tpl.make_dims(8192, 64, 8, 128, 28672, 80), 8)
    a = plan.workspace_size(1, 0)
    b = plan.workspace_size(4, 4096)
    c = plan.workspace_size(16, 8192)
    assert a < b < c
    assert c < 1 << 30


def test_gemv_option(tpl):
    plan = tpl.Plan(tpl.make_dims(256, 2, 2, 128, 688), 2)
    plan.set_option(tpl.TPL_OPT_GEMV_MODE, 2)
    plan.set_option(tpl.TPL_OPT_GEMV_MODE, 3)
    plan.set_option(tpl.TPL_OPT_GEMV_MODE, 4)
    plan.set_option(tpl.TPL_OPT_GEMV_MODE, 0)
    with pytest.raises(tpl.TplError):
        plan.set_option(tpl.TPL_OPT_GEMV_MODE, 5)
    with pytest.raises(tpl.TplError):
        plan.set_option(99, 0)


def test_prefill_tail_option(tpl):
    plan = tpl.Plan(tpl.make_dims(256, 2, 2, 128, 688), 2)
    plan.set_option(tpl.TPL_OPT_PREFILL_TAIL, 0)
    plan.set_option(tpl.TPL_OPT_PREFILL_TAIL, 1)
    for bad in (-1, 2):
        with pytest.raises(tpl.TplError):
            plan.set_option(tpl.TPL_OPT_PREFILL_TAIL, bad)


def test_prefill_chunk_validates_before_launch(tpl):
    """tpl_prefill_chunk's host checks: the chunk must fit the cache after its
    start position, the start must not be negative, fp32 plans are not
    supported, T = 0 does nothing."""
    plan = tpl.Plan(tpl.make_dims(256, 2, 2, 128, 688), 2)
    H = plan.handle
    fake = 1 << 20
    T = 16
    need = plan.prefill_workspace_size(T)
    kv = tpl.tpl_kv(fake, fake, 1, 40)
    args = lambda start, kvp=kv, ws_bytes=need, mode=0: (H, fake, ctypes.byref(kvp), fake, T, start, fake, None, fake,
                                                          ws_bytes, mode, None)
    assert tpl.tpl_prefill_chunk(*args(25)) == tpl.TPL_ENOMEM   # 25 + 16 > 40
    assert tpl.tpl_prefill_chunk(*args(-1)) == tpl.TPL_EINVAL
    assert tpl.tpl_prefill_chunk(*args(0, ws_bytes=need - 1)) == tpl.TPL_EWORKSPACE
    assert tpl.tpl_prefill_chunk(*args(0, mode=5)) == tpl.TPL_EINVAL
    assert tpl.tpl_prefill_chunk(H, fake, ctypes.byref(kv), fake, 0, 3, fake, None, fake, need, 0, None) == tpl.TPL_OK
    p32 = tpl.Plan(tpl.make_dims(256, 2, 2, 128, 688, 1, 1e-5, tpl.TPL_FP32_WEIGHTS), 2)
    assert tpl.tpl_prefill_chunk(p32.handle, fake, ctypes.byref(kv), fake, T, 0, fake, None, fake, need, 0,
                                 None) == tpl.TPL_EUNSUPPORTED


def test_rope_plan_workspace_and_maps_unchanged(tpl):
    """The rotation changes no layout: maps, packed size and workspace are
    those of the plan without it."""
    a = tpl.Plan(tpl.make_dims(1024, 16, 4, 128, 2816), 4)
    b = tpl.Plan(tpl.make_dims(1024, 16, 4, 128, 2816, 1, 1e-5, tpl.TPL_NORM | tpl.TPL_RESIDUAL | tpl.TPL_ROPE), 4)
    assert a.info().packed_layer_bytes == b.info().packed_layer_bytes
    for B, S in ((1, 0), (16, 4096), (64, 100)):
        assert a.workspace_size(B, S) == b.workspace_size(B, S)
    assert a.prefill_workspace_size(300) == b.prefill_workspace_size(300)
