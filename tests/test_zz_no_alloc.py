"""The allocation-free attention entry point, tpl_attn_decode_static.

It serves callers that cannot allocate device memory themselves (a plugin in
a host application that owns the whole device budget, a serving loop that
must never enter the allocator): it takes no workspace and keeps its split
partials in a fixed array of the library's static device memory.  These tests
call it through the C-ABI on two calls in a row and check it against the
oracle's attention output and, bit for bit, against tpl_attn_decode (which
uses a caller-provided workspace and chooses the same kernel).  The file is
collected last, and passes both alone in a fresh process and after the other
tests.
"""
import ctypes

import numpy as np
import pytest

from tests.conftest import has_gpu

pytestmark = pytest.mark.gpu


def _qkv(L):
    """q, k_new, v_new of the layer from the library's QKV step."""
    import torch
    d = L.dims
    q = torch.empty((L.B, d.n_q_heads, d.head_dim), dtype=torch.float32, device=L.x.device)
    kn = torch.empty((L.B, d.n_kv_heads, d.head_dim), dtype=torch.float32, device=L.x.device)
    vn = torch.empty_like(kn)
    L.plan.qkv(L.packed, L.kv, L.x, L.S, q, L.ws, kn, vn)
    return q, kn, vn


@pytest.mark.parametrize("case", [
    # H, nq, nkv, F, t, B, S: where the staged kernel runs (2*B*n_kv <= SMs)
    (1024, 16, 8, 2816, 8, 4, 700),
    # and where the register-streamed kernel runs (256 pairs x 2 > 148 SMs)
    (1024, 16, 8, 2816, 4, 16, 1000),
])
def test_attn_decode_static_matches_oracle_and_workspace_variant(gpu, case):
    import torch

    from megatron_tensor_transformer_plan_b200 import tpl
    from tests.gpu_util import TOL, assert_close_rel, make_layer, oracle_decode, to_np

    H, nq, nkv, F, t, B, S = case
    L = make_layer(H, nq, nkv, 128, F, t, B, S, seed=21)
    _, tr = oracle_decode(L)
    q, kn, vn = _qkv(L)
    o_ws = torch.empty((B, nq * 128), dtype=torch.bfloat16, device=gpu)
    L.plan.attn_decode(L.kv, q, S, o_ws, L.ws, kn, vn)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        o = torch.full_like(o_ws, float("nan"))
        rc = tpl.tpl_attn_decode_static(L.plan.handle, ctypes.byref(L.kv), q.data_ptr(), kn.data_ptr(),
                                        vn.data_ptr(), B, S, o.data_ptr(), stream)
        assert rc == tpl.TPL_OK, tpl.tpl_status_string(rc)
        torch.cuda.synchronize()
        assert_close_rel(to_np(o), tr["attn"], tol=TOL, what=f"static call {call} vs oracle")
        assert torch.equal(o, o_ws), f"static call {call} differs from tpl_attn_decode"
    assert L.plan.last_device_error() == tpl.TPL_OK


def test_attn_decode_static_stack_shape(gpu):
    """The attention step of the 70B-shaped stack (t = 8, batch 4, KV length
    4096) on seeded q / new k, v: two calls, each identical to the workspace
    call and close to it at the tolerance the two attention kernels keep."""
    import torch

    from megatron_tensor_transformer_plan_b200 import synth, tpl
    from tests.gpu_util import assert_close_rel, to_np

    H, nq, nkv, d, F, t, B, S = 8192, 64, 8, 128, 28672, 8, 4, 4096
    plan = tpl.Plan(tpl.make_dims(H, nq, nkv, d, F, 1), t)
    kl, vl = synth.kv_cache((B, nkv, S + 1, d), seed=7, device=gpu)
    k, v = plan.pack_kv(kl), plan.pack_kv(vl)
    kv = tpl.Plan.kv(k, v, B, S + 1)
    q = torch.empty((B, nq, d), dtype=torch.float32, device=gpu)
    synth.normal_(q, 1.8, seed=11)
    k_new = torch.empty((B, nkv, d), dtype=torch.float32, device=gpu)
    v_new = torch.empty_like(k_new)
    synth.normal_(k_new, 1.8, seed=12)
    synth.normal_(v_new, 1.8, seed=13)
    ws = plan.workspace(B, S, device=gpu)
    o_ref = torch.empty((B, nq * d), dtype=torch.bfloat16, device=gpu)
    plan.attn_decode(kv, q, S, o_ref, ws, k_new, v_new)
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        o = torch.full_like(o_ref, float("nan"))
        rc = tpl.tpl_attn_decode_static(plan.handle, ctypes.byref(kv), q.data_ptr(), k_new.data_ptr(),
                                        v_new.data_ptr(), B, S, o.data_ptr(), stream)
        assert rc == tpl.TPL_OK, tpl.tpl_status_string(rc)
        torch.cuda.synchronize()
        assert torch.equal(o, o_ref), f"static call {call} differs from tpl_attn_decode"
        assert_close_rel(to_np(o), to_np(o_ref), tol=8e-3, what=f"static call {call}")
    assert plan.last_device_error() == tpl.TPL_OK


def test_attn_decode_static_refuses_oversized_problem(gpu):
    """A problem whose split partials exceed the fixed scratch is refused
    before any launch.  Every buffer matches the descriptor it is passed
    with, so the refusal is not what keeps the call in bounds."""
    import torch

    from megatron_tensor_transformer_plan_b200 import tpl

    # 16 sequences x 64 kv heads = 1024 pairs, 16 query heads per kv head:
    # about 8.5 MB of split partials, above the 4 MiB array
    nq, nkv, d, B, S = 1024, 64, 128, 16, 128
    plan = tpl.Plan(tpl.make_dims(8192, nq, nkv, d, 28672, 1), 1)
    k = torch.zeros((1, B, nkv, S + 1, d), dtype=torch.bfloat16, device=gpu)
    v = torch.zeros_like(k)
    kv = tpl.Plan.kv(k, v, B, S + 1)
    q = torch.zeros((B, nq, d), dtype=torch.float32, device=gpu)
    o = torch.zeros((B, nq * d), dtype=torch.bfloat16, device=gpu)
    stream = torch.cuda.current_stream().cuda_stream
    rc = tpl.tpl_attn_decode_static(plan.handle, ctypes.byref(kv), q.data_ptr(), None, None, B, S, o.data_ptr(),
                                    stream)
    assert rc == tpl.TPL_ENOMEM, tpl.tpl_status_string(rc)
    torch.cuda.synchronize()
    assert np.all(o.cpu().float().numpy() == 0.0), "a refused call wrote its output"
